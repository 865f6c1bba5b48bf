"""Parity of the block-sparse (VSA fine attention) CUDA path --
attnqat_sparse_fwd / attnqat_sparse_bwd through the C ABI -- with the float64
oracle restricted to the same tile selection, and of the key-tile selection
attnqat_vsa_select with the oracle's (bit-exact: both rank in float32 with
the same fixed order of operations).

Bar: as for dense attention (relative L2 <= 1e-2, max-abs <= 5e-2 of the
oracle's RMS).  Rows of a query tile with no selected key tile must be exactly
O = 0, m = LSE = -inf, dQ = 0, and keys of a tile nobody selects exactly
dK = dV = 0.  With every tile selected the sparse path runs the dense kernels'
schedule on the same tiles, so its outputs must equal the dense call's bit for
bit."""
import numpy as np
import pytest

import oracle
import quantization_aware_attention_nvfp4_b200 as A
from quantization_aware_attention_nvfp4_b200 import workloads as W
from tests.helpers import assert_close, to_f64, to_gpu_bf16

pytestmark = pytest.mark.gpu


def _run_sparse(inp, mask, c, flags):
    import torch
    q, k, v, dO = (to_gpu_bf16(inp[n]) for n in ("q", "k", "v", "do"))
    tm = torch.from_numpy(mask).cuda()
    o, lse, m, ws = A.attnqat_sparse_fwd(q, k, v, tm, sm_scale=c, flags=flags)
    dq, dk, dv = A.attnqat_sparse_bwd(q, k, v, lse, m, dO, ws, tm, sm_scale=c, flags=flags)
    torch.cuda.synchronize()
    A.attnqat_device_status()
    return dict(o=o, lse=lse, m=m, dq=dq, dk=dk, dv=dv)


def _check_empty(got, mask, Lq, Lk):
    """Exact zeros / -inf where nothing is selected."""
    T = W.SPARSE_TILE
    o, lse, m, dq = (to_f64(got[n]) for n in ("o", "lse", "m", "dq"))
    dk, dv = to_f64(got["dk"]), to_f64(got["dv"])
    for b, h, i in zip(*np.nonzero(mask.sum(-1) == 0)):
        rows = slice(i * T, min((i + 1) * T, Lq))
        assert np.all(o[b, h, rows] == 0) and np.all(dq[b, h, rows] == 0)
        assert np.all(np.isneginf(lse[b, h, rows])) and np.all(np.isneginf(m[b, h, rows]))
    for b, h, j in zip(*np.nonzero(mask.sum(-2) == 0)):
        keys = slice(j * T, min((j + 1) * T, Lk))
        assert np.all(dk[b, h, keys] == 0) and np.all(dv[b, h, keys] == 0)


def _full_compare(w, mask, flags):
    inp = W.inputs(w)
    got = _run_sparse(inp, mask, w.sm_scale, flags)
    _check_empty(got, mask, w.Lq, w.Lk)
    ref = oracle.attention(inp["q"], inp["k"], inp["v"], w.sm_scale, flags, inp["do"], sel=mask,
                           tile=W.SPARSE_TILE)
    live = np.repeat(mask.sum(-1) > 0, W.SPARSE_TILE, axis=-1)[..., : w.Lq]  # rows with a selection
    for name, key in (("O", "o"), ("dQ", "dq")):
        assert_close(name, to_f64(got[key])[live], ref[name][live])
    assert_close("LSE", to_f64(got["lse"])[live], ref["lse"][live])
    assert_close("m", to_f64(got["m"])[live], ref["m"][live])
    assert_close("dK", to_f64(got["dk"]), ref["dK"])
    assert_close("dV", to_f64(got["dv"]), ref["dV"])


@pytest.mark.parametrize("Lq,Lk,D,flags", [
    (1000, 1100, 128, oracle.QUANT_ALL),
    (700, 1296, 128, oracle.QUANT_ALL),           # Lk % 32 == 16: the fp16 P V route
    (1000, 1100, 64, oracle.QUANT_ALL),
    (1000, 1100, 128, 0),
    (1000, 1100, 128, oracle.QUANT_Q | oracle.QUANT_K),
])
def test_random_selection_full(Lq, Lk, D, flags):
    """Random tile selection (about a third of the pairs) with ragged last
    query and key tiles, an empty query tile and an unselected key tile."""
    w = W.custom(1, 2, Lq, Lk, D, seed_index=800 + Lq % 89 + D + flags)
    mask = W.random_tile_mask(w, 0.35)
    mask[0, 0, 1, :] = 0            # a query tile with nothing selected
    mask[0, 1, :, 3] = 0            # a key tile nobody selects
    mask[0, 0, -1, -1] = 1          # the ragged corner
    _full_compare(w, mask, flags)


def test_one_key_tile_per_query_tile():
    w = W.custom(2, 1, 640, 640, 128, seed_index=811)
    nq = nk = 5
    mask = np.zeros((2, 1, nq, nk), np.uint8)
    mask[0, 0, np.arange(nq), np.arange(nq)] = 1            # diagonal
    mask[1, 0, np.arange(nq), (np.arange(nq) * 3 + 1) % nk] = 1
    _full_compare(w, mask, oracle.QUANT_ALL)


@pytest.mark.parametrize("Lq,Lk", [(1000, 1100), (256, 8192)])
def test_all_tiles_selected_equals_dense_bitwise(Lq, Lk):
    import torch
    w = W.custom(1, 2, Lq, Lk, 128, seed_index=812)
    inp = W.inputs(w)
    mask = np.ones((1, 2, -(-Lq // 128), -(-Lk // 128)), np.uint8)
    got = _run_sparse(inp, mask, w.sm_scale, oracle.QUANT_ALL)
    q, k, v, dO = (to_gpu_bf16(inp[n]) for n in ("q", "k", "v", "do"))
    o, lse, m, ws = A.attnqat_fwd(q, k, v, sm_scale=w.sm_scale)
    dq, dk, dv = A.attnqat_bwd(q, k, v, lse, m, dO, ws, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    for name, t in (("o", o), ("lse", lse), ("m", m), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert torch.equal(got[name], t), name


def test_tile_lists_past_one_warp():
    """More than 32 query and key tiles (the list builder's ballot loop runs
    several steps): a VSA-style top-k selection, sampled rows and blocks."""
    w = W.custom(1, 2, 4500, 4200, 128, seed_index=813)
    mask = W.tile_mask(w, 0.8)
    _sampled_compare(w, mask, heads=[(0, 0), (0, 1)], n_rows=48, n_blocks=48)


def _sampled_compare(w, mask, heads, n_rows, n_blocks, tag=""):
    """Sampled rows and 16-key blocks of the named heads against the oracle,
    plus properties on every head (finite; LSE >= m; LSE <= m + ln of the
    number of selected keys)."""
    inp = W.inputs(w)
    got = _run_sparse(inp, mask, w.sm_scale, oracle.QUANT_ALL)
    o, lse, m = to_f64(got["o"]), to_f64(got["lse"]), to_f64(got["m"])
    dq, dk, dv = to_f64(got["dq"]), to_f64(got["dk"]), to_f64(got["dv"])
    for name, arr in (("O", o), ("dQ", dq), ("dK", dk), ("dV", dv), ("LSE", lse)):
        assert np.all(np.isfinite(arr)), name
    assert np.all(lse >= m - 1e-4), "LSE >= m"
    nsel = np.repeat(mask.sum(-1), W.SPARSE_TILE, axis=-1)[..., : w.Lq] * W.SPARSE_TILE
    assert np.all(lse <= m + np.log(nsel) + 1e-3), "LSE <= m + ln(selected keys)"
    rng = np.random.default_rng(w.seed)
    nblk = (w.Lk + 15) // 16
    for (b, h) in heads:
        hd = oracle.Head(inp["q"][b, h], inp["k"][b, h], inp["v"][b, h], w.sm_scale, oracle.QUANT_ALL,
                         inp["do"][b, h], sel=mask[b, h], tile=W.SPARSE_TILE)
        rows = np.unique(np.concatenate([[0, w.Lq - 1], rng.choice(w.Lq, n_rows, replace=False)]))
        blocks = np.unique(np.concatenate([[0, nblk - 1], rng.choice(nblk, n_blocks, replace=False)]))
        O_r, lse_r, m_r, _ = hd.fwd_rows(rows)
        assert_close("O%s" % tag, o[b, h, rows], O_r)
        assert_close("LSE%s" % tag, lse[b, h, rows], lse_r)
        assert_close("dQ%s" % tag, dq[b, h, rows], hd.dq_rows(rows))
        dK_r, dV_r = hd.dkdv_blocks(blocks)
        keys = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
        valid = keys < w.Lk
        assert_close("dK%s" % tag, dk[b, h, keys[valid]], dK_r[valid])
        assert_close("dV%s" % tag, dv[b, h, keys[valid]], dV_r[valid])


@pytest.mark.slow
def test_vsa_wan_6h_31200_sparsity_09_sampled():
    """The timed sparse workload: H6 L31200 D128, 25 of 244 key tiles per
    query tile (sparsity 0.9)."""
    w = W.get("wan_6h_31200")
    _sampled_compare(w, W.tile_mask(w, 0.9), heads=[(0, 0), (0, w.H - 1)], n_rows=48, n_blocks=48,
                     tag=" vsa")


@pytest.mark.parametrize("B,H,Lq,Lk,D,topk", [
    (1, 2, 1000, 1100, 128, 3),
    (2, 1, 300, 700, 64, 2),
    (1, 1, 130, 90, 128, 5),        # topk above the tile count: every tile
    (1, 6, 31200, 31200, 128, 25),  # the pages' shape at sparsity 0.9
])
def test_vsa_select_matches_oracle(B, H, Lq, Lk, D, topk):
    import torch
    w = W.custom(B, H, Lq, Lk, D, seed_index=820 + D + topk)
    inp = W.inputs(w, with_grad=False)
    q, k = to_gpu_bf16(inp["q"]), to_gpu_bf16(inp["k"])
    mask = A.attnqat_vsa_select(q, k, topk)
    torch.cuda.synchronize()
    got = mask.cpu().numpy()
    for b in range(B):
        for h in range(H):
            want, _ = oracle.vsa_select(inp["q"][b, h], inp["k"][b, h], topk, tile=W.SPARSE_TILE)
            assert np.array_equal(got[b, h], want), (b, h)
    assert np.all(got.sum(-1) == min(topk, got.shape[-1]))


def test_selection_feeds_sparse_attention():
    """The whole VSA fine path: attnqat_vsa_select's mask into the sparse
    forward and backward, against the oracle run on the oracle's own mask."""
    import torch
    w = W.custom(1, 2, 900, 1000, 128, seed_index=830)
    inp = W.inputs(w)
    q, k = to_gpu_bf16(inp["q"]), to_gpu_bf16(inp["k"])
    topk = W.topk_tiles(-(-w.Lk // W.SPARSE_TILE), 0.7)
    mask = A.attnqat_vsa_select(q, k, topk).cpu().numpy()
    want = np.stack([np.stack([oracle.vsa_select(inp["q"][0, h], inp["k"][0, h], topk)[0] for h in range(2)])])
    assert np.array_equal(mask, want)
    _full_compare(w, want, oracle.QUANT_ALL)
