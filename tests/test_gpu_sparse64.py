"""The tile-64 profile of block-sparse attention (ATTNQAT_TILE64 on
attnqat_sparse_fwd / attnqat_sparse_bwd, attnqat_vsa_select_tiles with
tile = 64) through the C ABI, against the float64 oracle restricted to the same
64-token block selection.

The kernels run 128 x 128 tiles whose list entries carry the four 64 x 64
quadrants a tile pair selects; these tests cover rows whose 64-token block
selects nothing inside a listed tile (O = 0, m = LSE = -inf, dQ = 0 exactly),
key blocks nobody selects (dK = dV = 0 exactly), ragged last blocks, the flag
sets, both head dimensions, bitwise agreement with the dense call when every
block is selected and with the 128-token path when the selection is whole
128-token tiles, and the selection kernel at 64-token tiles bit for bit."""
import numpy as np
import pytest

import oracle
import quantization_aware_attention_nvfp4_b200 as A
from quantization_aware_attention_nvfp4_b200 import workloads as W
from tests.helpers import assert_close, to_f64, to_gpu_bf16

pytestmark = pytest.mark.gpu

T = 64


def _run(inp, mask, c, flags, tile=T):
    import torch
    q, k, v, dO = (to_gpu_bf16(inp[n]) for n in ("q", "k", "v", "do"))
    tm = torch.from_numpy(np.ascontiguousarray(mask)).cuda()
    o, lse, m, ws = A.attnqat_sparse_fwd(q, k, v, tm, sm_scale=c, flags=flags, tile=tile)
    dq, dk, dv = A.attnqat_sparse_bwd(q, k, v, lse, m, dO, ws, tm, sm_scale=c, flags=flags, tile=tile)
    torch.cuda.synchronize()
    A.attnqat_device_status()
    return dict(o=o, lse=lse, m=m, dq=dq, dk=dk, dv=dv)


def _random_mask(w, p, seed):
    rng = np.random.default_rng([w.seed, 300, seed])
    return (rng.random((w.B, w.H, -(-w.Lq // T), -(-w.Lk // T))) < p).astype(np.uint8)


def _full_compare(w, mask, flags):
    inp = W.inputs(w)
    got = _run(inp, mask, w.sm_scale, flags)
    o, lse, m, dq = (to_f64(got[n]) for n in ("o", "lse", "m", "dq"))
    dk, dv = to_f64(got["dk"]), to_f64(got["dv"])
    for b, h, i in zip(*np.nonzero(mask.sum(-1) == 0)):
        rows = slice(i * T, min((i + 1) * T, w.Lq))
        assert np.all(o[b, h, rows] == 0) and np.all(dq[b, h, rows] == 0), "empty query block"
        assert np.all(np.isneginf(lse[b, h, rows])) and np.all(np.isneginf(m[b, h, rows]))
    for b, h, j in zip(*np.nonzero(mask.sum(-2) == 0)):
        keys = slice(j * T, min((j + 1) * T, w.Lk))
        assert np.all(dk[b, h, keys] == 0) and np.all(dv[b, h, keys] == 0), "unselected key block"
    ref = oracle.attention(inp["q"], inp["k"], inp["v"], w.sm_scale, flags, inp["do"], sel=mask, tile=T)
    live = np.repeat(mask.sum(-1) > 0, T, axis=-1)[..., : w.Lq]
    for name, key in (("O", "o"), ("dQ", "dq")):
        assert_close(name, to_f64(got[key])[live], ref[name][live])
    assert_close("LSE", lse[live], ref["lse"][live])
    assert_close("m", m[live], ref["m"][live])
    assert_close("dK", dk, ref["dK"])
    assert_close("dV", dv, ref["dV"])


@pytest.mark.parametrize("Lq,Lk,D,flags", [
    (1000, 1100, 128, oracle.QUANT_ALL),
    (700, 1296, 128, oracle.QUANT_ALL),           # Lk % 32 == 16: the fp16 P V route
    (1000, 1100, 64, oracle.QUANT_ALL),
    (1000, 1100, 128, 0),
    (1000, 1100, 128, oracle.QUANT_Q | oracle.QUANT_K),
    (300, 200, 64, oracle.QUANT_V | oracle.QUANT_P),
])
def test_random_block_selection_full(Lq, Lk, D, flags):
    """Random 64-token block selection (about a third of the pairs) with
    ragged last blocks, a query block with nothing selected whose partner in
    the same 128-token tile selects something, and an unselected key block."""
    w = W.custom(1, 2, Lq, Lk, D, seed_index=830 + Lq % 89 + D + flags)
    mask = _random_mask(w, 0.35, flags + D)
    mask[0, 0, 2, :] = 0            # query block 2 (rows 128..191): nothing
    mask[0, 0, 3, :4] = 1           # ... while block 3 of the same 128-row tile selects
    mask[0, 1, :, min(5, mask.shape[3] - 2)] = 0   # a key block nobody selects
    mask[0, 0, -1, -1] = 1          # the ragged corner
    _full_compare(w, mask, flags)


def test_diagonal_quadrants():
    """Each query block attends only its own key block: the selected quadrant
    of a 128-token tile pair is on its diagonal, the other two in the pair
    stay masked."""
    w = W.custom(1, 1, 512, 512, 128, seed_index=840)
    nb = 512 // T
    mask = np.zeros((1, 1, nb, nb), np.uint8)
    mask[0, 0, np.arange(nb), np.arange(nb)] = 1
    _full_compare(w, mask, oracle.QUANT_ALL)


def test_every_block_selected_equals_dense_bitwise():
    import torch
    w = W.custom(1, 2, 1000, 1100, 128, seed_index=841)
    inp = W.inputs(w)
    mask = np.ones((1, 2, -(-w.Lq // T), -(-w.Lk // T)), np.uint8)
    got = _run(inp, mask, w.sm_scale, oracle.QUANT_ALL)
    q, k, v, dO = (to_gpu_bf16(inp[n]) for n in ("q", "k", "v", "do"))
    o, lse, m, ws = A.attnqat_fwd(q, k, v, sm_scale=w.sm_scale)
    dq, dk, dv = A.attnqat_bwd(q, k, v, lse, m, dO, ws, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    for name, t in (("o", o), ("lse", lse), ("m", m), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert torch.equal(got[name], t), name


def test_whole_tile_selection_equals_the_128_token_path_bitwise():
    """A 64-token mask that selects whole 128-token tiles gives the 128-token
    path's results bit for bit."""
    import torch
    w = W.custom(1, 2, 1000, 1100, 128, seed_index=842)
    inp = W.inputs(w)
    m128 = W.random_tile_mask(w, 0.4)
    m64 = np.repeat(np.repeat(m128, 2, axis=2), 2, axis=3)[..., : -(-w.Lq // T), : -(-w.Lk // T)]
    a = _run(inp, m64, w.sm_scale, oracle.QUANT_ALL, tile=64)
    b = _run(inp, m128, w.sm_scale, oracle.QUANT_ALL, tile=128)
    for name in ("o", "lse", "m", "dq", "dk", "dv"):
        assert torch.equal(a[name], b[name]), name


@pytest.mark.parametrize("B,H,Lq,Lk,D,topk", [(1, 2, 1000, 1100, 128, 5), (2, 1, 300, 4000, 64, 7),
                                             (1, 1, 130, 70, 128, 9)])
def test_vsa_select_at_64_token_tiles_bitwise(B, H, Lq, Lk, D, topk):
    import torch
    w = W.custom(B, H, Lq, Lk, D, seed_index=850 + Lq % 31)
    inp = W.inputs(w, with_grad=False)
    q, k = to_gpu_bf16(inp["q"]), to_gpu_bf16(inp["k"])
    got = A.attnqat_vsa_select(q, k, topk, tile=T).cpu().numpy()
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            want, _ = oracle.vsa_select(inp["q"][b, h], inp["k"][b, h], topk, tile=T)
            assert np.array_equal(got[b, h], want), (b, h)


def test_vsa_select_score_rows_in_global_memory_bitwise():
    """More than 2048 key tiles (Lk = 131200 at 64-token tiles: 2050): the
    top-k kernel works on its score row in global memory instead of a
    shared-memory copy.  Bit for bit against the oracle."""
    import torch
    w = W.custom(1, 1, 300, 131200, 64, seed_index=860)
    inp = W.inputs(w, with_grad=False)
    q, k = to_gpu_bf16(inp["q"]), to_gpu_bf16(inp["k"])
    assert -(-w.Lk // T) > 2048
    got = A.attnqat_vsa_select(q, k, 37, tile=T).cpu().numpy()
    torch.cuda.synchronize()
    want, _ = oracle.vsa_select(inp["q"][0, 0], inp["k"][0, 0], 37, tile=T)
    assert np.array_equal(got[0, 0], want)
    assert np.all(got.sum(-1) == 37)


@pytest.mark.slow
def test_pages_shape_at_sparsity_09_sampled():
    """H6 L31200 with the tile-64 selection at sparsity 0.9 (49 of 488 key
    blocks per query block), sampled rows and key blocks of two heads."""
    import torch
    w = W.get("wan_6h_31200")
    inp = W.inputs(w)
    q, k = to_gpu_bf16(inp["q"]), to_gpu_bf16(inp["k"])
    nk = -(-w.Lk // T)
    topk = W.topk_tiles(nk, 0.9)
    mask = A.attnqat_vsa_select(q, k, topk, tile=T).cpu().numpy()
    torch.cuda.synchronize()
    got = _run(inp, mask, w.sm_scale, oracle.QUANT_ALL)
    o, lse, m = to_f64(got["o"]), to_f64(got["lse"]), to_f64(got["m"])
    dq, dk, dv = to_f64(got["dq"]), to_f64(got["dk"]), to_f64(got["dv"])
    for arr in (o, dq, dk, dv, lse):
        assert np.all(np.isfinite(arr))
    rng = np.random.default_rng(860)
    for h in (0, w.H - 1):
        hd = oracle.Head(inp["q"][0, h], inp["k"][0, h], inp["v"][0, h], w.sm_scale, oracle.QUANT_ALL,
                         inp["do"][0, h], sel=mask[0, h], tile=T)
        rows = np.unique(np.concatenate([[0, w.Lq - 1], rng.choice(w.Lq, 48, replace=False)]))
        O_r, lse_r, _, _ = hd.fwd_rows(rows)
        assert_close("O", o[0, h, rows], O_r)
        assert_close("LSE", lse[0, h, rows], lse_r)
        assert_close("dQ", dq[0, h, rows], hd.dq_rows(rows))
        nblk = (w.Lk + 15) // 16
        blocks = np.unique(np.concatenate([[0, nblk - 1], rng.choice(nblk, 40, replace=False)]))
        dK_r, dV_r = hd.dkdv_blocks(blocks)
        keys = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
        valid = keys < w.Lk
        assert_close("dK", dk[0, h, keys[valid]], dK_r[valid])
        assert_close("dV", dv[0, h, keys[valid]], dV_r[valid])
