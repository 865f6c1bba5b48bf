"""Bit-exact parity of the standalone NVFP4 quantizer (attnqat_quantize)
against the float64 oracle: FP4 codes and E4M3 scale bytes identical, and the
dequantized bf16 values identical bit for bit."""
import numpy as np
import pytest

import oracle
from quantization_aware_attention_nvfp4_b200 import workloads as W
from tests.helpers import bf16_bits, to_gpu_bf16

pytestmark = pytest.mark.gpu


def _gpu_quantize(bits2d):
    import quantization_aware_attention_nvfp4_b200 as A
    x = to_gpu_bf16(bits2d)
    codes, scales, deq = A.attnqat_quantize(x)
    return codes.cpu().numpy(), scales.cpu().numpy(), bf16_bits(deq)


def _oracle_deq_bits(deq_f64):
    # the oracle's dequantized values are exact in bf16: round-trip is exact
    return W.f32_to_bf16_bits(deq_f64.astype(np.float32))


def _check(bits2d):
    rows, cols = bits2d.shape
    c_gpu, s_gpu, d_gpu = _gpu_quantize(bits2d)
    c_ref, s_ref, d_ref = oracle.quantize_rows(bits2d, rows, cols, cols, 1)
    assert np.array_equal(s_gpu, s_ref), np.argwhere(s_gpu != s_ref)[:5]
    assert np.array_equal(c_gpu, c_ref), np.argwhere(c_gpu != c_ref)[:5]
    assert np.array_equal(d_ref.astype(np.float32).astype(np.float64), d_ref)
    assert np.array_equal(d_gpu, _oracle_deq_bits(d_ref))


def test_every_finite_bf16_as_block_amax():
    """Each finite bf16 value once as the amax of its own block, with random
    partners at or below it (covers every scale code, subnormal scales, zero
    scales and saturation)."""
    rng = np.random.default_rng(101)
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = W.bf16_bits_to_f32(bits)
    keep = np.isfinite(vals)
    bits, vals = bits[keep], vals[keep]
    blocks = rng.uniform(-1, 1, (bits.size, 16)).astype(np.float32) * np.abs(vals)[:, None]
    b = W.f32_to_bf16_bits(blocks)
    b[:, 0] = bits
    _check(b)


def _e4m3_positive():
    """The 126 positive finite E4M3 values (4 exponent bits, bias 7, 3
    mantissa bits; 448 the largest)."""
    v = [m / 8 * 2.0 ** -6 for m in range(1, 8)]
    v += [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if not (e == 15 and m == 7)]
    return v


def test_every_bf16_value_under_every_scale():
    """Every pair of a block scale and an element value the code conversion
    can meet: for each positive E4M3 scale s, blocks whose amax is exactly
    6 s (so the scale is s) and whose other 15 elements run through every bf16
    value of magnitude <= 6 s, both signs (280649 blocks)."""
    pos_bits = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)  # every finite bf16 >= 0
    pos_vals = (pos_bits.astype(np.uint32) << 16).view(np.float32)
    blocks = []
    for s in _e4m3_positive():
        a = np.array([6.0 * s], np.float32)
        a_bits = np.uint16(a.view(np.uint32)[0] >> 16)
        assert float((np.uint32(a_bits) << 16).view(np.float32)) == 6.0 * s  # exact in bf16
        sel = pos_bits[pos_vals <= a[0]]
        vals = np.concatenate([sel, sel | np.uint16(0x8000)])
        vals = np.concatenate([vals, np.zeros((-len(vals)) % 15, np.uint16)]).reshape(-1, 15)
        blocks.append(np.concatenate([np.full((len(vals), 1), a_bits, np.uint16), vals], axis=1))
    _check(np.ascontiguousarray(np.concatenate(blocks)))


def test_tie_rich_and_edge_blocks():
    rng = np.random.default_rng(102)
    e4m3 = np.array([oracle.e4m3_value(c) for c in range(127)])
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for sc in range(1, 127):
        s = e4m3[sc]
        for _ in range(8):
            x = rng.choice(mids, 16) * s * rng.choice([-1, 1], 16)
            x[0] = 6 * s
            rows.append(x.astype(np.float32))
    rows.append(np.full(16, 3000.0, np.float32))
    rows.append(np.array([-0.0, 0.0] * 8, np.float32))
    rows.append(np.array([-1e-30] + [1.0] * 15, np.float32))
    for a in (3.02, 3.2, 3.49, 0.5, 2.99):  # subnormal-scale neighbourhood
        x = np.zeros(16, np.float32)
        x[0] = a * 2 ** -9
        rows.append(x)
    b = np.stack([W.f32_to_bf16_bits(r) for r in rows])
    _check(b)


@pytest.mark.parametrize("rows,cols,scale", [(4096, 128, 1.0), (513, 64, 30.0), (7, 16, 1e-3)])
def test_random_rows(rows, cols, scale):
    rng = np.random.default_rng(rows + cols)
    x = (rng.standard_normal((rows, cols)) * scale).astype(np.float32)
    _check(W.f32_to_bf16_bits(x))


def test_transposed_view_blocks_along_tokens():
    """V blocked along tokens: the [BH, D, Lk] view of a [BH, Lk, D] tensor."""
    import quantization_aware_attention_nvfp4_b200 as A
    rng = np.random.default_rng(103)
    BH, Lk, D = 3, 272, 128
    v = W.f32_to_bf16_bits(rng.standard_normal((BH, Lk, D)).astype(np.float32))
    vt = to_gpu_bf16(v).transpose(1, 2)  # [BH, D, Lk], strides (Lk*D, 1, D)
    codes, scales, deq = A.attnqat_quantize(vt)
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    deq_bits = bf16_bits(deq.transpose(1, 2))  # back to [BH, Lk, D]
    for z in range(BH):
        c_ref, s_ref, d_ref = oracle.quantize_rows(v[z], D, Lk, 1, D)
        assert np.array_equal(scales[z], s_ref)
        assert np.array_equal(codes[z], c_ref)
        assert np.array_equal(deq_bits[z], _oracle_deq_bits(d_ref.T))


def test_rejects_bad_arguments():
    import torch
    import quantization_aware_attention_nvfp4_b200 as A
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(A.AttnQatError) as e:
        A.attnqat_quantize(x)
    assert e.value.status == A.EINVAL


# ------------------------------------------ NVFP4 with an FP32 global scale ----

def _check_gs(bits, batch, rows, cols, sb, sr, sc, view):
    """GPU global-scale quantizer vs the oracle on one strided view."""
    import quantization_aware_attention_nvfp4_b200 as A
    codes, scales, deq, g = A.attnqat_quantize_gs(view)
    # the oracle quantizes each batch slice of the same view; G is global, so
    # fold the batch into rows: rows of every slice share one max
    flat_rows = []
    for z in range(batch):
        for r in range(rows):
            flat_rows.append(bits.reshape(-1)[z * sb + r * sr + np.arange(cols) * sc])
    flat = np.stack(flat_rows).astype(np.uint16)
    c_ref, s_ref, d_ref, g_ref = oracle.quantize_rows_gs(flat, batch * rows, cols, cols, 1)
    assert np.float32(g.item()) == np.float32(g_ref)
    assert np.array_equal(scales.cpu().numpy().reshape(batch * rows, -1), s_ref)
    assert np.array_equal(codes.cpu().numpy().reshape(batch * rows, -1), c_ref)
    # bf16_bits makes deq contiguous in the view's logical order [batch, rows, cols]
    assert np.array_equal(bf16_bits(deq).reshape(batch * rows, cols), d_ref)


@pytest.mark.parametrize("mag", [1.0, 1e-6, 3e3, 1e-30, 0.0])
def test_global_scale_rows(mag):
    """Random rows across magnitudes (a huge G for tiny tensors, G = 1 for an
    all-zero one), plus a block far below the tensor max."""
    rng = np.random.default_rng(int(abs(np.log10(mag))) if mag else 5)
    x = rng.standard_normal((96, 128)).astype(np.float32) * np.float32(mag)
    x[7, :16] *= np.float32(1e-4)
    bits = W.f32_to_bf16_bits(x)
    _check_gs(bits, 1, 96, 128, 0, 128, 1, to_gpu_bf16(bits))


def test_global_scale_g_one_and_overflow():
    """max|x| = 2688 (G = 1: the plain format) and a max below 2688 / FLT_MAX
    (G saturates to the largest finite float32)."""
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((32, 64)) * 200).astype(np.float32)
    x[3, 9] = -2688.0
    bits = W.f32_to_bf16_bits(x)
    _check_gs(bits, 1, 32, 64, 0, 64, 1, to_gpu_bf16(bits))
    tiny = np.zeros((4, 32), np.uint16)
    tiny[1, 5] = 3      # subnormal bf16 values only
    tiny[2, 17] = 0x8001
    _check_gs(tiny, 1, 4, 32, 0, 32, 1, to_gpu_bf16(tiny))


def test_global_scale_batched_transposed_view():
    """V-like view: per head, channels as rows and tokens as columns (blocks
    of 16 tokens), one global scale over all heads."""
    rng = np.random.default_rng(13)
    BH, L, D = 3, 96, 64
    x = rng.standard_normal((BH, L, D)).astype(np.float32)
    bits = W.f32_to_bf16_bits(x).reshape(BH, L, D)
    t = to_gpu_bf16(bits)
    view = t.transpose(-1, -2)  # [BH, D, L] with strides (L*D, 1, D)
    _check_gs(bits, BH, D, L, L * D, 1, D, view)
