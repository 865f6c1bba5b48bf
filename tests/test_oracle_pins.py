"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle against brute force, exact rational arithmetic,
torch's own float8 conversion, closed forms, invariants, or autograd /
finite differences of an independently written straight-through surrogate.
A plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong tie rule) fails at least one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from quantization_aware_attention_nvfp4_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = W.bf16_bits_to_f32(bits)
    keep = np.isfinite(vals)
    return bits[keep], vals[keep].astype(np.float64)


# ------------------------------------------------------------ E4M3 scale ----

def test_e4m3_value_table_matches_torch():
    codes = np.arange(127, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_value(int(c)) for c in codes])
    assert np.array_equal(ref, mine)


def test_e4m3_scale_exhaustive_vs_torch_float8():
    """(i) every finite bf16 amax: scale = nearest E4M3 to a/6 (torch's RNE
    float32 -> float8_e4m3fn conversion, saturated at 448)."""
    _, vals = _all_finite_bf16()
    a = np.abs(vals)
    t = np.minimum(a / 6.0, 448.0).astype(np.float32)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_round_div6(x) for x in a], dtype=np.uint8)
    bad = np.nonzero(ref != mine)[0]
    assert bad.size == 0, (a[bad[:5]], ref[bad[:5]], mine[bad[:5]])


def _e4m3_values_fraction():
    out = []
    for code in range(127):
        e, m = code >> 3, code & 7
        out.append(Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7))
    return out


def _nearest_fraction(target, values):
    """Brute force: the nearest of the sorted values, ties to the even index,
    saturating to the last."""
    if target >= values[-1]:
        return len(values) - 1
    best = None
    for i, v in enumerate(values):
        d = abs(v - target)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def test_e4m3_scale_rational_bruteforce_sample():
    """Exact rational arithmetic, independent of float64 and of torch."""
    vals = _e4m3_values_fraction()
    rng = np.random.default_rng(7)
    bits, fv = _all_finite_bf16()
    pick = rng.choice(np.nonzero((np.abs(fv) < 3000) & (fv != 0))[0], 400, replace=False)
    # plus every exact tie a = 6 * midpoint that bf16 can represent
    ties = []
    for i in range(126):
        mid = (vals[i] + vals[i + 1]) / 2 * 6
        f = float(mid)
        if Fraction(f) == mid and W.f32_to_bf16_bits(np.array([f], np.float32))[0] is not None:
            b = W.f32_to_bf16_bits(np.array([f], np.float32))
            if Fraction(float(W.bf16_bits_to_f32(b)[0])) == mid:
                ties.append(f)
    assert len(ties) > 50
    for a in list(np.abs(fv[pick])) + ties:
        want = _nearest_fraction(Fraction(float(a)) / 6, vals)
        assert oracle.e4m3_round_div6(float(a)) == want, a


def test_e4m3_golden_points():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_e2m1_points.json")))
    for code, v in g["e4m3_value_of_code"]:
        assert oracle.e4m3_value(code) == v
    for a, code in g["e4m3_amax_to_code"]:
        assert oracle.e4m3_round_div6(a) == code, a


# ------------------------------------------------------------- E2M1 code ----

def _e2m1_thresholds(ax, s):
    """Independent formulation: count the midpoints passed.  Crossing the
    midpoint between codes k and k+1 needs a strict '>' when k is even (the
    tie stays on the even k) and '>=' when k is odd (the tie moves up to the
    even k+1)."""
    code = np.zeros(ax.shape, np.int32)
    for k in range(7):
        mid2 = (GRID[k] + GRID[k + 1]) * s
        if k % 2 == 0:
            code += (2 * ax > mid2)
        else:
            code += (2 * ax >= mid2)
    return code


def test_e2m1_exhaustive_all_bf16_times_all_scales():
    """(ii) every finite bf16 x against every positive finite E4M3 scale."""
    _, fv = _all_finite_bf16()
    ax = np.abs(fv)
    for sc in range(1, 127):
        s = oracle.e4m3_value(sc)
        mine = oracle.e2m1_round_many(ax, np.float64(s))
        ref = _e2m1_thresholds(ax, s)
        bad = np.nonzero(mine != ref)[0]
        assert bad.size == 0, (sc, ax[bad[:5]], mine[bad[:5]], ref[bad[:5]])


def test_e2m1_golden_points():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_e2m1_points.json")))
    assert [oracle.e2m1_value(c) for c in range(8)] == g["e2m1_grid"]
    for ratio, code in g["e2m1_ratio_to_code"]:
        assert oracle.e2m1_round(ratio, 1.0) == code, ratio
        assert oracle.e2m1_round(ratio * 0.171875, 0.171875) == code, ratio


# ------------------------------------------------------- block quantizer ----

def _fq_block_fraction(xs):
    """Pure-Python exact fq of one block (Fractions): returns (codes, scale
    code, dequantized Fractions)."""
    vals = _e4m3_values_fraction()
    grid = [Fraction(g) for g in GRID]
    fx = [Fraction(float(x)) for x in xs]
    a = max(abs(x) for x in fx)
    sc = 0 if a == 0 else _nearest_fraction(a / 6, vals)
    s = vals[sc]
    codes, deq = [], []
    for x, raw in zip(fx, xs):
        neg = 1 if np.signbit(raw) else 0
        c = 0 if s == 0 else _nearest_fraction(abs(x) / s, grid)
        codes.append((neg << 3) | c)
        deq.append((-1 if neg else 1) * grid[c] * s)
    return codes, sc, deq


def _special_blocks(rng):
    """Random, tie-rich, subnormal-scale, saturating and signed-zero blocks."""
    blocks = []
    for _ in range(60):
        blocks.append(rng.standard_normal(16).astype(np.float32) * np.float32(10 ** rng.uniform(-4, 3)))
    vals = [float(v) for v in _e4m3_values_fraction()]
    for _ in range(60):  # elements exactly at g*s midpoints of a normal scale
        sc = int(rng.integers(8, 120))
        s = vals[sc]
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
        x = rng.choice(mids, 16) * s * rng.choice([-1, 1], 16)
        x[0] = 6 * s  # pins the scale at s
        blocks.append(x.astype(np.float32))
    for _ in range(30):  # tiny blocks: subnormal or zero scales
        blocks.append(rng.uniform(-1, 1, 16).astype(np.float32) * np.float32(rng.uniform(0.002, 0.2)))
    blocks.append(np.full(16, 3000.0, np.float32))  # saturating scale
    blocks.append(np.array([-0.0, 0.0] * 8, np.float32))  # zero block, signed zeros
    blocks.append(np.array([-1e-30] + [1.0] * 15, np.float32))  # negative to zero -> 0x8
    return blocks


def test_block_quantizer_vs_exact_rationals():
    rng = np.random.default_rng(11)
    blocks = _special_blocks(rng)
    bits = np.stack([W.f32_to_bf16_bits(b) for b in blocks])
    codes, scales, deq = oracle.quantize_rows(bits, len(blocks), 16, 16, 1)
    for r, b in enumerate(bits):
        xs = W.bf16_bits_to_f32(b)
        want_codes, want_sc, want_deq = _fq_block_fraction(xs)
        assert scales[r, 0] == want_sc
        packed = [want_codes[2 * i] | (want_codes[2 * i + 1] << 4) for i in range(8)]
        assert list(codes[r]) == packed, r
        assert [Fraction(float(v)) for v in deq[r]] == want_deq


def test_block_quantizer_strided_view_and_packing():
    """A transposed view (blocks along tokens, stride D) equals quantizing the
    explicitly transposed array; codes put element 2i in the low nibble."""
    rng = np.random.default_rng(3)
    L, D = 64, 32
    x = W.f32_to_bf16_bits(rng.standard_normal((L, D)).astype(np.float32))
    c1, s1, d1 = oracle.quantize_rows(x, D, L, 1, D)  # rows = channels, cols = tokens
    xt = np.ascontiguousarray(x.T)
    c2, s2, d2 = oracle.quantize_rows(xt, D, L, L, 1)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2) and np.array_equal(d1, d2)
    lo = c1 & 0xF
    hi = c1 >> 4
    mag = np.array(GRID)
    s = np.array([[oracle.e4m3_value(int(v)) for v in row] for row in s1])
    for r in range(D):
        for j in range(L):
            code = lo[r, j // 2] if j % 2 == 0 else hi[r, j // 2]
            val = mag[code & 7] * s[r, j // 16] * (-1 if code & 8 else 1)
            assert val == d1[r, j]


def test_sign_symmetry():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((500, 64)).astype(np.float32) * np.float32(3)
    b = W.f32_to_bf16_bits(x)
    nb = W.f32_to_bf16_bits(-x)
    _, s1, d1 = oracle.quantize_rows(b, 500, 64, 64, 1)
    _, s2, d2 = oracle.quantize_rows(nb, 500, 64, 64, 1)
    assert np.array_equal(s1, s2)
    assert np.array_equal(d1, -d2)


def test_idempotence_on_normal_scales():
    """fq(fq(x)) == fq(x) whenever the block scale is a normal E4M3 (>= 2^-6):
    the block max then lands on code 6, so the rescale reproduces s."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((4000, 16)) * 10 ** rng.uniform(-1.5, 2.5, (4000, 1))
    b = W.f32_to_bf16_bits(x.astype(np.float32))
    _, sc, d1 = oracle.quantize_rows(b, 4000, 16, 16, 1)
    normal = sc[:, 0] >= 8
    assert normal.sum() > 3500
    d2, sc2 = oracle.fq_f64_rows(d1)
    assert np.array_equal(d2[normal], d1[normal])
    assert np.array_equal(sc2[normal], sc[normal])


def test_idempotence_predicted_failures_on_subnormal_scales():
    """Single-element blocks a*[1,0,...]: with a in (3, 3.5]*2^-9 the scale is
    2^-9 (a/6 just above half of 2^-9), the element rounds to 3*2^-9, and a
    second pass sees a/6 = 0.5*2^-9, a tie that goes to scale 0."""
    for a in [3.02 * 2 ** -9, 3.2 * 2 ** -9, 3.49 * 2 ** -9]:
        x = np.zeros((1, 16))
        x[0, 0] = a
        b = W.f32_to_bf16_bits(x.astype(np.float32))
        _, sc, d1 = oracle.quantize_rows(b, 1, 16, 16, 1)
        assert sc[0, 0] == 1 and d1[0, 0] == 3 * 2 ** -9
        d2, sc2 = oracle.fq_f64_rows(d1)
        assert sc2[0, 0] == 0 and np.all(d2 == 0)


# ---------------------------------------------------------- attention ------

def _rand_bits(rng, shape, scale=1.0):
    return W.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _f(bits):
    return W.bf16_bits_to_f32(bits).astype(np.float64)


def test_unquantized_forward_matches_sdpa_and_softmax():
    rng = np.random.default_rng(21)
    B, H, Lq, Lk, D = 1, 2, 40, 48, 32
    q, k, v = (_rand_bits(rng, (B, H, L, D)) for L in (Lq, Lk, Lk))
    c = 0.3
    out = oracle.attention(q, k, v, c, flags=0)
    qt, kt, vt = (torch.from_numpy(_f(x)) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=c).numpy()
    assert np.max(np.abs(out["O"] - ref)) < 1e-12
    # second formulation: explicit softmax in float64 numpy
    S = np.einsum("bhid,bhjd->bhij", _f(q), _f(k)) * c
    P = np.exp(S - S.max(-1, keepdims=True))
    P /= P.sum(-1, keepdims=True)
    assert np.allclose(P.sum(-1), 1.0, atol=1e-14)
    assert np.max(np.abs(out["O"] - P @ _f(v))) < 1e-12
    assert np.max(np.abs(out["m"] - S.max(-1))) < 1e-13
    assert np.max(np.abs(np.exp(out["lse"]) - np.exp(S).sum(-1)) / np.exp(S).sum(-1)) < 1e-13


def test_probabilities_sum_to_one():
    """With V = 1 (unquantized) and quant_p off, O = sum_j P_ij = 1 for every
    row.  (fq would move a block of ones to 6 * E4M3(1/6) = 1.03125.)"""
    rng = np.random.default_rng(22)
    q = _rand_bits(rng, (1, 1, 33, 16), 2.0)
    k = _rand_bits(rng, (1, 1, 64, 16), 2.0)
    v = W.f32_to_bf16_bits(np.ones((1, 1, 64, 16), np.float32))
    out = oracle.attention(q, k, v, 0.5, flags=oracle.QUANT_Q | oracle.QUANT_K)
    assert np.max(np.abs(out["O"] - 1.0)) < 1e-14
    out = oracle.attention(q, k, v, 0.5, flags=oracle.QUANT_Q | oracle.QUANT_K | oracle.QUANT_V)
    assert np.max(np.abs(out["O"] - 1.03125)) < 1e-14


def test_identical_keys_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "identical_keys.json")))
    rng = np.random.default_rng(23)
    Lq, Lk, D = 20, 64, 32
    q = _rand_bits(rng, (1, 1, Lq, D))
    krow = _rand_bits(rng, (1, 1, 1, D))
    k = np.repeat(krow, Lk, axis=2)
    v = _rand_bits(rng, (1, 1, Lk, D))
    _, _, vdeq = oracle.quantize_rows(v[0, 0], D, Lk, 1, D)  # fq(V) blocks along tokens
    vmean = vdeq.T.mean(0)
    out = oracle.attention(q, k, v, 0.125, flags=oracle.QUANT_ALL)
    assert oracle.e4m3_round_div6(1.0) == g["scale_code"]
    assert oracle.e4m3_value(g["scale_code"]) == g["scale_value"]
    assert np.max(np.abs(out["O"][0, 0] - g["p_hat_constant"] * vmean)) < 1e-14
    out2 = oracle.attention(q, k, v, 0.125, flags=oracle.QUANT_ALL & ~oracle.QUANT_P)
    assert np.max(np.abs(out2["O"][0, 0] - vmean)) < 1e-14


def test_single_block_lk16_matches_bruteforce():
    """Lk = 16: one P block; everything written out by hand with Fractions
    for the fq of P~ and float64 elsewhere."""
    rng = np.random.default_rng(24)
    Lq, Lk, D = 8, 16, 16
    q, k, v = _rand_bits(rng, (1, 1, Lq, D)), _rand_bits(rng, (1, 1, Lk, D)), _rand_bits(rng, (1, 1, Lk, D))
    c = 0.25
    out = oracle.attention(q, k, v, c, flags=oracle.QUANT_ALL)
    _, _, qd = oracle.quantize_rows(q[0, 0], Lq, D, D, 1)
    _, _, kd = oracle.quantize_rows(k[0, 0], Lk, D, D, 1)
    _, _, vd = oracle.quantize_rows(v[0, 0], D, Lk, 1, D)
    vd = vd.T
    for i in range(Lq):
        S = np.array([c * sum(qd[i, d] * kd[j, d] for d in range(D)) for j in range(Lk)])
        Pt = np.exp(S - S.max())
        _, _, ph = _fq_block_fraction(Pt)
        ph = np.array([float(x) for x in ph])
        O = ph @ vd / Pt.sum()
        assert np.max(np.abs(out["O"][0, 0, i] - O)) < 1e-12


def test_ragged_lk_zero_padding_equivalence():
    """Lk not a multiple of 16: zero-padding K/V rows to the next block and
    masking them out gives the same O (padded keys get P~ = 0)."""
    rng = np.random.default_rng(25)
    Lq, Lk, D = 10, 40, 16
    q, k, v = _rand_bits(rng, (1, 1, Lq, D)), _rand_bits(rng, (1, 1, Lk, D)), _rand_bits(rng, (1, 1, Lk, D))
    hd = oracle.Head(q[0, 0], k[0, 0], v[0, 0], 0.3, oracle.QUANT_ALL)
    O, lse, m, l = hd.fwd_rows()
    # by hand with the oracle's own operands, padding to 48 with exp(-inf) = 0
    S = hd.Qh @ hd.Kh.T * 0.3
    Pt = np.exp(S - S.max(1, keepdims=True))
    Ptp = np.concatenate([Pt, np.zeros((Lq, 8))], 1)
    Ph, _ = oracle.fq_f64_rows(Ptp)
    O2 = Ph[:, :Lk] @ hd.Vh / Pt.sum(1, keepdims=True)
    assert np.max(np.abs(O - O2)) < 1e-13


# ------------------------------------------------------------ gradients ----

def _torch_attention_grads(q, k, v, dO, c):
    qt, kt, vt = (torch.tensor(_f(x), requires_grad=True) for x in (q, k, v))
    S = qt @ kt.transpose(-1, -2) * c
    O = torch.softmax(S, -1) @ vt
    (O * torch.tensor(_f(dO))).sum().backward()
    return O.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def test_unquantized_gradients_match_autograd():
    rng = np.random.default_rng(31)
    Lq, Lk, D = 24, 32, 16
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for L in (Lq, Lk, Lk, Lq))
    c = 0.4
    out = oracle.attention(q, k, v, c, flags=0, do_bits=dO)
    O, gq, gk, gv = _torch_attention_grads(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], c)
    for name, ref in (("dQ", gq), ("dK", gk), ("dV", gv)):
        assert np.max(np.abs(out[name][0, 0] - ref)) < 1e-12, name


def test_unquantized_gradients_central_differences():
    rng = np.random.default_rng(32)
    Lq, Lk, D = 6, 16, 8
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for L in (Lq, Lk, Lk, Lq))
    c = 0.7
    out = oracle.attention(q, k, v, c, flags=0, do_bits=dO)
    base = {n: _f(x)[0, 0] for n, x in (("q", q), ("k", k), ("v", v))}
    g = _f(dO)[0, 0]

    def loss(vals):
        S = vals["q"] @ vals["k"].T * c
        P = np.exp(S - S.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        return float(np.sum((P @ vals["v"]) * g))

    h = 1e-6
    for name, grad in (("q", out["dQ"]), ("k", out["dK"]), ("v", out["dV"])):
        for idx in [(0, 0), (1, 3), (3, 7)]:
            plus = {n: a.copy() for n, a in base.items()}
            minus = {n: a.copy() for n, a in base.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            assert abs(fd - grad[0, 0][idx]) < 1e-7, (name, idx)


@pytest.mark.parametrize("flag", [oracle.QUANT_Q, oracle.QUANT_K, oracle.QUANT_V])
def test_single_quantizer_equals_quantizing_that_operand_first(flag):
    """One quantizer on its own is plain attention on that operand's fq copy:
    fq(Q), fq(K) in blocks of 16 along D, fq(V) in blocks of 16 tokens per
    channel from token 0, each taken from the block quantizer (pinned above
    against exact rationals; its values are exact in bf16).  Forward and
    straight-through gradients against torch's float64 softmax attention
    and autograd on those copies.  A quantizer keyed to the wrong flag bit,
    or fq(V) blocked along channels, fails this."""
    rng = np.random.default_rng(60 + flag)
    Lq, Lk, D = 24, 48, 32
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for L in (Lq, Lk, Lk, Lq))
    c = 0.35
    pre = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
    name = {oracle.QUANT_Q: "q", oracle.QUANT_K: "k", oracle.QUANT_V: "v"}[flag]
    x = pre[name][0, 0]
    if name == "v":
        _, _, deq = oracle.quantize_rows(x, D, Lk, 1, D)  # the [D, Lk] view: blocks along tokens
        deq = deq.T
    else:
        _, _, deq = oracle.quantize_rows(x, x.shape[0], D, D, 1)
    fq_bits = W.f32_to_bf16_bits(deq.astype(np.float32))
    assert np.array_equal(_f(fq_bits), deq)  # exact in bf16
    pre[name] = fq_bits.reshape(1, 1, -1, D)
    out = oracle.attention(q, k, v, c, flags=flag, do_bits=dO)
    O, gq, gk, gv = _torch_attention_grads(pre["q"][0, 0], pre["k"][0, 0], pre["v"][0, 0], dO[0, 0], c)
    for key, ref in (("O", O), ("dQ", gq), ("dK", gk), ("dV", gv)):
        assert np.max(np.abs(out[key][0, 0] - ref)) < 1e-12, key


def _ste_surrogate_grads(hd, q, k, v, dO, c, flags):
    """Gradient of the straight-through surrogate by torch autograd.

    The offsets d_X = fq(X0) - X0 (X in Q, K, V), d_P = fq(P~0) - P~0 and the
    row max m0 are frozen at the base point; then
        O(Q, K, V) = (P~ + d_P)(V + d_V) / l,  P~ = exp((Q + d_Q)(K + d_K)^T c - m0),
        l = sum_j P~.
    Its exact gradient is what the straight-through estimator prescribes."""
    Q0, K0, V0 = (_f(x)[0, 0] for x in (q, k, v))
    dQo, dKo, dVo = hd.Qh - Q0, hd.Kh - K0, hd.Vh - V0
    S0 = hd.Qh @ hd.Kh.T * c
    m0 = S0.max(1, keepdims=True)
    Pt0 = np.exp(S0 - m0)
    if flags & oracle.QUANT_P:
        Ph0, _ = oracle.fq_f64_rows(Pt0)
    else:
        Ph0 = Pt0
    dPo = Ph0 - Pt0
    qt, kt, vt = (torch.tensor(a, requires_grad=True) for a in (Q0, K0, V0))
    Pt = torch.exp((qt + torch.tensor(dQo)) @ (kt + torch.tensor(dKo)).T * c - torch.tensor(m0))
    l = Pt.sum(1, keepdim=True)
    O = (Pt + torch.tensor(dPo)) @ (vt + torch.tensor(dVo)) / l
    (O * torch.tensor(_f(dO)[0, 0])).sum().backward()
    return O.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("flags", [oracle.QUANT_ALL, oracle.QUANT_Q | oracle.QUANT_K,
                                   oracle.QUANT_V | oracle.QUANT_P])
def test_quantized_gradients_match_ste_surrogate(flags):
    rng = np.random.default_rng(33 + flags)
    Lq, Lk, D = 20, 48, 32
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for L in (Lq, Lk, Lk, Lq))
    c = 0.35
    out = oracle.attention(q, k, v, c, flags=flags, do_bits=dO)
    hd = oracle.Head(q[0, 0], k[0, 0], v[0, 0], c, flags, dO[0, 0])
    O, gq, gk, gv = _ste_surrogate_grads(hd, q, k, v, dO, c, flags)
    assert np.max(np.abs(out["O"][0, 0] - O)) < 1e-12
    for name, ref in (("dQ", gq), ("dK", gk), ("dV", gv)):
        err = np.max(np.abs(out[name][0, 0] - ref))
        assert err < 1e-11, (name, err)


def test_quantized_gradients_finite_differences_of_surrogate():
    """Central differences of the frozen-offset surrogate (float64 numpy),
    independent of autograd."""
    rng = np.random.default_rng(41)
    Lq, Lk, D = 8, 32, 16
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for L in (Lq, Lk, Lk, Lq))
    c, flags = 0.5, oracle.QUANT_ALL
    out = oracle.attention(q, k, v, c, flags=flags, do_bits=dO)
    hd = oracle.Head(q[0, 0], k[0, 0], v[0, 0], c, flags, dO[0, 0])
    Q0, K0, V0 = (_f(x)[0, 0] for x in (q, k, v))
    off = {"q": hd.Qh - Q0, "k": hd.Kh - K0, "v": hd.Vh - V0}
    S0 = hd.Qh @ hd.Kh.T * c
    m0 = S0.max(1, keepdims=True)
    Pt0 = np.exp(S0 - m0)
    dP = oracle.fq_f64_rows(Pt0)[0] - Pt0
    g = _f(dO)[0, 0]

    def loss(vals):
        Pt = np.exp((vals["q"] + off["q"]) @ (vals["k"] + off["k"]).T * c - m0)
        return float(np.sum(((Pt + dP) @ (vals["v"] + off["v"]) / Pt.sum(1, keepdims=True)) * g))

    base = {"q": Q0, "k": K0, "v": V0}
    h = 1e-6
    for name, grad in (("q", out["dQ"]), ("k", out["dK"]), ("v", out["dV"])):
        for idx in [(0, 0), (2, 5), (7, 15)]:
            plus = {n: a.copy() for n, a in base.items()}
            minus = {n: a.copy() for n, a in base.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            assert abs(fd - grad[0, 0][idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx, fd)


def test_dv_literal_reading_zeroes_normalised_blocks():
    """The literal fq(P~/l) reading: with no global scale the normalised blocks
    of a long row have amax/6 below half the smallest E4M3 subnormal, so every
    block flushes to zero and dV vanishes (why it is not the default)."""
    rng = np.random.default_rng(51)
    Lq, Lk, D = 4, 4096, 16
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D), 0.1) for L in (Lq, Lk, Lk, Lq))
    out = oracle.attention(q, k, v, 0.25, flags=oracle.QUANT_ALL | oracle.DV_QUANT_NORMALIZED,
                           do_bits=dO)
    assert np.all(out["dV"] == 0)
    out2 = oracle.attention(q, k, v, 0.25, flags=oracle.QUANT_ALL, do_bits=dO)
    assert np.max(np.abs(out2["dV"])) > 0
    assert np.array_equal(out["dK"], out2["dK"]) and np.array_equal(out["dQ"], out2["dQ"])


def test_sampled_rows_equal_full_computation():
    """The row/block sampling entry points agree with the full computation."""
    rng = np.random.default_rng(61)
    Lq, Lk, D = 40, 64, 16
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for L in (Lq, Lk, Lk, Lq))
    hd = oracle.Head(q[0, 0], k[0, 0], v[0, 0], 0.3, oracle.QUANT_ALL, dO[0, 0])
    dQ, dK, dV = hd.backward()
    rows = np.array([3, 17, 39])
    O, lse, m, l = hd.fwd_rows(rows)
    st = hd.stats()
    assert np.array_equal(O, st["O"][rows])
    assert np.array_equal(hd.dq_rows(rows), dQ[rows])
    dKs, dVs = hd.dkdv_blocks(np.array([2]))
    assert np.array_equal(dKs, dK[32:48]) and np.array_equal(dVs, dV[32:48])


# ------------------------------------------- block-sparse fine attention ----
# VSA fine attention (vsqa-test-1.3b metadata.json, "attention": backend
# VSA_QAT_TRAIN_C128, 128-token cubes, selected key blocks per query block,
# NVFP4 fake-quant on the fine branch).  The oracle takes the selection as a
# tile mask; small tiles (multiples of 16) keep these pins fast.

def _sparse_case(seed, Lq, Lk, D, T, p=0.5):
    rng = np.random.default_rng(seed)
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for L in (Lq, Lk, Lk, Lq))
    nqt, nkt = -(-Lq // T), -(-Lk // T)
    sel = (rng.random((nqt, nkt)) < p).astype(np.uint8)
    return q, k, v, dO, sel


def test_sparse_all_tiles_selected_is_dense():
    q, k, v, dO, _ = _sparse_case(71, 70, 90, 32, 32)
    sel = np.ones((1, 1, 3, 3), np.uint8)
    a = oracle.attention(q, k, v, 0.2, oracle.QUANT_ALL, dO, sel=sel, tile=32)
    b = oracle.attention(q, k, v, 0.2, oracle.QUANT_ALL, dO)
    for key in b:
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("flags", [oracle.QUANT_ALL, 0, oracle.QUANT_V | oracle.QUANT_P])
def test_sparse_equals_dense_attention_on_the_gathered_tiles(flags):
    """Each query tile's output and dQ equal dense attention of its rows
    against the concatenation of its selected key tiles (the oracle's dense
    path, pinned above); dK, dV equal the sum of those per-tile gradients;
    a query tile with no selection gives O = 0, LSE = m = -inf, dQ = 0; an
    unselected key tile gets dK = dV = 0.  Tiles are whole 16-blocks (the
    ragged last key tile comes last in the gather), so fq(V) and fq(P~) see
    the same blocks either way."""
    Lq, Lk, D, T = 100, 150, 32, 32
    q, k, v, dO, sel = _sparse_case(72 + flags, Lq, Lk, D, T)
    sel[1, :] = 0          # a query tile with nothing selected
    sel[:, 2] = 0          # a key tile nobody selects
    sel[0, 4] = sel[3, 4] = 1  # the ragged last key tile, from the ragged last query tile too
    sel[2, 0] = 1
    c = 0.21
    sp = oracle.attention(q, k, v, c, flags, dO, sel=sel[None, None], tile=T)
    dK = np.zeros((Lk, D))
    dV = np.zeros((Lk, D))
    for I in range(sel.shape[0]):
        rows = np.arange(I * T, min((I + 1) * T, Lq))
        js = np.nonzero(sel[I])[0]
        if js.size == 0:
            assert np.all(sp["O"][0, 0, rows] == 0) and np.all(sp["dQ"][0, 0, rows] == 0)
            assert np.all(np.isneginf(sp["lse"][0, 0, rows])) and np.all(np.isneginf(sp["m"][0, 0, rows]))
            continue
        keys = np.concatenate([np.arange(J * T, min((J + 1) * T, Lk)) for J in js])
        hd = oracle.Head(q[0, 0, rows], k[0, 0, keys], v[0, 0, keys], c, flags, dO[0, 0, rows])
        st = hd.stats()
        dQg, dKg, dVg = hd.backward()
        assert np.max(np.abs(sp["O"][0, 0, rows] - st["O"])) <= 1e-12 * np.max(np.abs(st["O"]))
        assert np.max(np.abs(sp["lse"][0, 0, rows] - st["lse"])) <= 1e-12
        assert np.array_equal(sp["m"][0, 0, rows], st["m"])
        assert np.max(np.abs(sp["dQ"][0, 0, rows] - dQg)) <= 1e-11 * np.max(np.abs(dQg))
        dK[keys] += dKg
        dV[keys] += dVg
    assert np.all(sp["dK"][0, 0, 64:96] == 0) and np.all(sp["dV"][0, 0, 64:96] == 0)
    assert np.max(np.abs(sp["dK"][0, 0] - dK)) <= 1e-11 * np.max(np.abs(dK))
    assert np.max(np.abs(sp["dV"][0, 0] - dV)) <= 1e-11 * np.max(np.abs(dV))


def test_sparse_quantizers_off_vs_torch_masked_sdpa():
    """Quantizers off: block-sparse attention is softmax attention under the
    token mask the tile selection expands to (torch's masked SDPA and
    autograd, float64)."""
    Lq, Lk, D, T = 80, 112, 16, 16
    q, k, v, dO, sel = _sparse_case(73, Lq, Lk, D, T, p=0.3)
    sel[np.arange(sel.shape[0]), np.arange(sel.shape[0]) % sel.shape[1]] = 1  # no empty row
    c = 0.37
    mask = np.kron(sel, np.ones((T, T), np.uint8))[:Lq, :Lk].astype(bool)
    qt, kt, vt = (torch.tensor(_f(x[0, 0]), requires_grad=True) for x in (q, k, v))
    O = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None],
                                                         attn_mask=torch.tensor(mask)[None], scale=c)[0]
    (O * torch.tensor(_f(dO[0, 0]))).sum().backward()
    sp = oracle.attention(q, k, v, c, 0, dO, sel=sel[None, None], tile=T)
    for name, ref in (("O", O.detach()), ("dQ", qt.grad), ("dK", kt.grad), ("dV", vt.grad)):
        ref = ref.numpy()
        assert np.max(np.abs(sp[name][0, 0] - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref))), name


# ----------------------------------------------------- causal masking ----

def test_causal_quantizers_off_vs_torch_sdpa():
    """Quantizers off: causal attention is torch's causal SDPA (float64
    autograd for the gradients)."""
    rng = np.random.default_rng(95)
    L, D, c = 48, 16, 0.31
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for _ in range(4))
    qt, kt, vt = (torch.tensor(_f(x[0, 0]), requires_grad=True) for x in (q, k, v))
    O = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], is_causal=True, scale=c)[0]
    (O * torch.tensor(_f(dO[0, 0]))).sum().backward()
    out = oracle.attention(q, k, v, c, oracle.CAUSAL, dO)
    for name, ref in (("O", O.detach()), ("dQ", qt.grad), ("dK", kt.grad), ("dV", vt.grad)):
        ref = ref.numpy()
        assert np.max(np.abs(out[name][0, 0] - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref))), name


def test_causal_rows_equal_dense_attention_on_their_prefix():
    """With fq on: row i of causal attention is dense attention of row i
    against keys 0..i (fq(P~)'s ragged last block is zero-padded there, as the
    masked keys are zeros here); fq(V) runs on the whole V in both (its
    blocks along tokens do not depend on the mask), so the prefix problems
    take the oracle's fq(V) as plain bf16 input.  dK, dV sum the prefix
    problems' gradients."""
    rng = np.random.default_rng(96)
    L, D, c = 40, 16, 0.27
    q, k, v, dO = (_rand_bits(rng, (1, 1, L, D)) for _ in range(4))
    flags = oracle.QUANT_ALL | oracle.CAUSAL
    out = oracle.attention(q, k, v, c, flags, dO)
    vh = oracle.Head(q[0, 0], k[0, 0], v[0, 0], c, oracle.QUANT_ALL).Vh
    vq = W.f32_to_bf16_bits(vh.astype(np.float32))
    assert np.array_equal(W.bf16_bits_to_f32(vq).astype(np.float64), vh)
    pre = oracle.QUANT_ALL & ~oracle.QUANT_V
    dK = np.zeros((L, D))
    dV = np.zeros((L, D))
    for i in range(L):
        hd = oracle.Head(q[0, 0, i:i + 1], k[0, 0, : i + 1], vq[: i + 1], c, pre, dO[0, 0, i:i + 1])
        st = hd.stats()
        dQi, dKi, dVi = hd.backward()
        assert np.max(np.abs(out["O"][0, 0, i] - st["O"][0])) <= 1e-12 * np.max(np.abs(st["O"]))
        assert abs(out["lse"][0, 0, i] - st["lse"][0]) <= 1e-12 and out["m"][0, 0, i] == st["m"][0]
        assert np.max(np.abs(out["dQ"][0, 0, i] - dQi[0])) <= 1e-11 * max(np.max(np.abs(dQi)), 1e-30)
        dK[: i + 1] += dKi
        dV[: i + 1] += dVi
    assert np.max(np.abs(out["dK"][0, 0] - dK)) <= 1e-11 * np.max(np.abs(dK))
    assert np.max(np.abs(out["dV"][0, 0] - dV)) <= 1e-11 * np.max(np.abs(dV))


def test_causal_needs_equal_lengths():
    rng = np.random.default_rng(97)
    q, k = _rand_bits(rng, (8, 16)), _rand_bits(rng, (12, 16))
    with pytest.raises(ValueError):
        oracle.Head(q, k, k, 0.3, oracle.CAUSAL)


# ----------------------------------------------- sparse block selection ----

def test_vsa_select_agrees_with_float64_ranking():
    """Coarse scores within float32 rounding of the float64 tile-mean dot
    products, and the kept set equal to the float64 top-k wherever the k-th
    and (k+1)-th float64 scores are apart by more than the rounding."""
    rng = np.random.default_rng(91)
    Lq, Lk, D, T, topk = 300, 700, 64, 32, 5
    q, k = _rand_bits(rng, (Lq, D)), _rand_bits(rng, (Lk, D))
    mask, scores = oracle.vsa_select(q, k, topk, tile=T)
    qf, kf = _f(q), _f(k)
    qm = np.stack([qf[i:i + T].mean(0) for i in range(0, Lq, T)])
    km = np.stack([kf[j:j + T].mean(0) for j in range(0, Lk, T)])
    s64 = qm @ km.T
    assert np.max(np.abs(scores - s64)) <= 1e-5 * np.max(np.abs(s64))
    checked = 0
    for i in range(s64.shape[0]):
        order = np.argsort(-s64[i], kind="stable")
        if s64[i, order[topk - 1]] - s64[i, order[topk]] > 1e-4 * np.max(np.abs(s64)):
            want = np.zeros(s64.shape[1], np.uint8)
            want[order[:topk]] = 1
            assert np.array_equal(mask[i], want), i
            checked += 1
        assert mask[i].sum() == topk
    assert checked >= s64.shape[0] - 1


def test_vsa_select_ties_go_to_the_lower_tile_and_topk_bounds():
    """Constant tiles: score = D * a_J exactly; equal scores keep the lower
    key tile; topk = 1 is the argmax, topk >= the tile count keeps all."""
    D, T = 16, 16
    a = [1.0, 3.0, 3.0, 2.0, 3.0]
    k = W.f32_to_bf16_bits(np.repeat(np.array(a, np.float32), T)[:, None] * np.ones((1, D), np.float32))
    q = W.f32_to_bf16_bits(np.ones((T, D), np.float32))
    mask, scores = oracle.vsa_select(q, k, 2, tile=T)
    assert np.array_equal(scores[0], np.array(a, np.float32) * D)
    assert np.array_equal(mask[0], [0, 1, 1, 0, 0])
    assert np.array_equal(oracle.vsa_select(q, k, 1, tile=T)[0][0], [0, 1, 0, 0, 0])
    assert np.all(oracle.vsa_select(q, k, 9, tile=T)[0] == 1)


def test_vsa_select_ragged_tile_mean_uses_its_valid_rows():
    """A ragged last key tile is averaged over its valid rows only: five rows
    of 7 beat full tiles of 3 (zero-padding would average them to 2.19)."""
    D, T = 16, 16
    vals = np.concatenate([np.full(2 * T, 3.0), np.full(5, 7.0)]).astype(np.float32)
    k = W.f32_to_bf16_bits(vals[:, None] * np.ones((1, D), np.float32))
    q = W.f32_to_bf16_bits(np.ones((T, D), np.float32))
    mask, scores = oracle.vsa_select(q, k, 1, tile=T)
    assert np.array_equal(mask[0], [0, 0, 1]) and scores[0, 2] == 7.0 * D


# ------------------------------------------ NVFP4 with an FP32 global scale ----

def _bf16_value_fraction(h):
    return Fraction(float(W.bf16_bits_to_f32(np.array([h], np.uint16))[0]))


def _bf16_rne_fraction(v):
    """bf16 bit pattern nearest to the exact rational v >= 0, ties to the even
    pattern (a search over neighbouring patterns in exact arithmetic)."""
    if v == 0:
        return 0
    h = int(W.f32_to_bf16_bits(np.array([float(v)], np.float32))[0])
    while h > 0 and _bf16_value_fraction(h) > v:
        h -= 1
    while _bf16_value_fraction(h + 1) <= v:
        h += 1
    lo, hi = _bf16_value_fraction(h), _bf16_value_fraction(h + 1)
    if v - lo != hi - v:
        return h if v - lo < hi - v else h + 1
    return h if h % 2 == 0 else h + 1


def _fq_gs_fraction(xs):
    """The global-scale format in exact rationals: G = float32(2688 / max|x|),
    block scale = nearest E4M3 to a_b G / 6, code = nearest E2M1 to |x| G / s,
    value = sign * E2M1 * s / G rounded to bf16 (all ties to even)."""
    amax = float(np.max(np.abs(xs)))
    g32 = np.float32(1.0) if amax == 0 else np.float32(2688.0) / np.float32(amax)
    if not np.isfinite(g32):
        g32 = np.float32(np.finfo(np.float32).max)
    g = Fraction(float(g32))
    vals = _e4m3_values_fraction()
    grid = [Fraction(v) for v in GRID]
    rows, cols = xs.shape
    codes = np.zeros((rows, cols), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    deq = np.zeros((rows, cols), np.uint16)
    for r in range(rows):
        for b in range(cols // 16):
            blk = [Fraction(float(v)) for v in xs[r, 16 * b:16 * b + 16]]
            k = _nearest_fraction(max(abs(v) for v in blk) * g / 6, vals)
            s = vals[k]
            scales[r, b] = k
            for i, v in enumerate(blk):
                neg = 1 if np.signbit(xs[r, 16 * b + i]) else 0
                c = 0 if s == 0 else _nearest_fraction(abs(v) * g / s, grid)
                codes[r, 16 * b + i] = (neg << 3) | c
                deq[r, 16 * b + i] = _bf16_rne_fraction(grid[c] * s / g) | (0x8000 if neg else 0)
    return codes, scales, deq, float(g32)


def _pack(codes):
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("seed,mag", [(1, 1.0), (2, 1e-5), (3, 3e3), (4, 0.37), (5, 1e-30)])
def test_global_scale_format_vs_exact_rationals(seed, mag):
    """Exact rational brute force of the global-scale format on random and
    tie-rich tensors across magnitudes (including tiny ones whose global
    scale is huge)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((6, 32)).astype(np.float32) * np.float32(mag)
    x[1, :16] *= np.float32(1e-3)          # a block far below the tensor max
    x[2, :] = np.float32(0.0)              # zero blocks
    bits = W.f32_to_bf16_bits(x)
    xs = W.bf16_bits_to_f32(bits).reshape(6, 32)
    codes, scales, deq, g = oracle.quantize_rows_gs(bits, 6, 32, 32, 1)
    wc, ws, wd, wg = _fq_gs_fraction(xs)
    assert np.float32(g) == np.float32(wg)
    assert np.array_equal(scales, ws)
    assert np.array_equal(codes, _pack(wc))
    assert np.array_equal(deq, wd)


def test_global_scale_one_reduces_to_plain_format():
    """max|x| = 2688 gives G = 1: codes, scales and values of the plain
    format (pinned above against torch and exact rationals)."""
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((5, 48)) * 300).astype(np.float32)
    x[3, 7] = -2688.0
    bits = W.f32_to_bf16_bits(x)
    c, s, d, g = oracle.quantize_rows_gs(bits, 5, 48, 48, 1)
    c0, s0, d0 = oracle.quantize_rows(bits, 5, 48, 48, 1)
    assert g == 1.0
    assert np.array_equal(c, c0) and np.array_equal(s, s0)
    assert np.array_equal(W.bf16_bits_to_f32(d.reshape(-1)).astype(np.float64), d0.reshape(-1))


@pytest.mark.parametrize("k", [-6, -1, 3, 9])
def test_global_scale_power_of_two_is_plain_format_of_scaled_input(k):
    """max|x| = 2688 * 2^-k gives G = 2^k exactly, and the result is the plain
    format applied to x * 2^k, scaled back by 2^-k."""
    rng = np.random.default_rng(20 + k)
    x = (rng.standard_normal((4, 64)) * 100).astype(np.float32)
    x[0, 0] = 2688.0
    x = x * np.float32(2.0 ** -k)
    bits = W.f32_to_bf16_bits(x)
    c, s, d, g = oracle.quantize_rows_gs(bits, 4, 64, 64, 1)
    assert g == 2.0 ** k
    xs = W.bf16_bits_to_f32(bits).reshape(4, 64) * np.float32(2.0 ** k)
    c0, s0, d0 = oracle.quantize_rows(W.f32_to_bf16_bits(xs), 4, 64, 64, 1)
    assert np.array_equal(c, c0) and np.array_equal(s, s0)
    assert np.array_equal(W.bf16_bits_to_f32(d.reshape(-1)).astype(np.float64) * 2.0 ** k, d0.reshape(-1))


def test_global_max_round_trips_and_sign_symmetry():
    """The tensor's largest magnitude gets scale 448 and code 6 and comes back
    exactly; fq(-x) = -fq(x) with the same scales and global scale."""
    rng = np.random.default_rng(31)
    for trial in range(20):
        x = (rng.standard_normal((3, 32)) * 10 ** rng.uniform(-8, 4)).astype(np.float32)
        bits = W.f32_to_bf16_bits(x)
        xs = W.bf16_bits_to_f32(bits).reshape(3, 32)
        c, s, d, g = oracle.quantize_rows_gs(bits, 3, 32, 32, 1)
        i = np.unravel_index(np.argmax(np.abs(xs)), xs.shape)
        assert s[i[0], i[1] // 16] == 126  # E4M3 448
        assert W.bf16_bits_to_f32(d[i[0], i[1]:i[1] + 1])[0] == xs[i]
        cn, sn, dn, gn = oracle.quantize_rows_gs(bits ^ np.uint16(0x8000), 3, 32, 32, 1)
        assert gn == g and np.array_equal(sn, s)
        assert np.array_equal(cn, c ^ np.uint8(0x88)) and np.array_equal(dn, d ^ np.uint16(0x8000))


def test_global_scale_sees_every_element():
    """G comes from the largest magnitude anywhere in the view: planted at each
    corner (and inside) of a row-major tensor, and at the last element of a
    transposed (strided) view, the largest magnitude M gives G =
    float32(2688 / M)."""
    rng = np.random.default_rng(41)
    rows, cols = 5, 48
    base = (rng.standard_normal((rows, cols)) * 0.5).astype(np.float32)
    for r, c in [(0, 0), (0, cols - 1), (rows - 1, 0), (rows - 1, cols - 1), (2, 17)]:
        for big in (np.float32(-37.0), np.float32(9984.0)):  # both exact in bf16
            x = base.copy()
            x[r, c] = big
            bits = W.f32_to_bf16_bits(x)
            _, _, _, g = oracle.quantize_rows_gs(bits, rows, cols, cols, 1)
            assert np.float32(g) == np.float32(2688.0) / np.abs(big), (r, c, big)
    # rows of the view = the 3 columns of a [16, 3] tensor (element (r, j) at
    # x[j, r]); the largest magnitude is the view's last element
    x16 = (rng.standard_normal((16, 3)) * 0.5).astype(np.float32)
    x16[15, 2] = np.float32(-99.0)
    _, _, _, g16 = oracle.quantize_rows_gs(W.f32_to_bf16_bits(x16), 3, 16, 1, 3)
    assert np.float32(g16) == np.float32(2688.0) / np.float32(99.0)


def test_global_scale_special_cases():
    """All-zero input: G = 1 and zeros; a max below 2688 / FLT_MAX: the
    quotient overflows float32 and G saturates to the largest finite float."""
    z = np.zeros((2, 16), np.uint16)
    c, s, d, g = oracle.quantize_rows_gs(z, 2, 16, 16, 1)
    assert g == 1.0 and not c.any() and not s.any() and not d.any()
    assert oracle.global_scale(0.0) == 1.0
    tiny = float(W.bf16_bits_to_f32(np.array([1], np.uint16))[0])  # smallest bf16 subnormal
    assert oracle.global_scale(tiny) == float(np.finfo(np.float32).max)
    assert oracle.global_scale(2688.0) == 1.0
