"""No kernel writes outside its buffers: every output (o, lse, m, dq, dk, dv)
and the workspace sit inside canary guard bands (tests/helpers.guarded), for
dense, block-sparse (with an empty query tile and ragged tiles) and causal
calls; the guarded run's outputs equal an ordinary run's bit for bit (the
kernels are deterministic)."""
import pytest

import oracle
import quantization_aware_attention_nvfp4_b200 as A
from quantization_aware_attention_nvfp4_b200 import workloads as W
from tests.helpers import guarded, guards_intact, to_gpu_bf16

pytestmark = pytest.mark.gpu


def _call(mode, q, k, v, dO, c, flags, tm, outs=None, ws=None):
    o_out = None if outs is None else outs[:3]
    g_out = None if outs is None else outs[3:]
    if mode == "sparse":
        o, lse, m, ws = A.attnqat_sparse_fwd(q, k, v, tm, sm_scale=c, flags=flags, ws=ws, out=o_out)
        dq, dk, dv = A.attnqat_sparse_bwd(q, k, v, lse, m, dO, ws, tm, sm_scale=c, flags=flags, out=g_out)
    else:
        o, lse, m, ws = A.attnqat_fwd(q, k, v, sm_scale=c, flags=flags, ws=ws, out=o_out)
        dq, dk, dv = A.attnqat_bwd(q, k, v, lse, m, dO, ws, sm_scale=c, flags=flags, out=g_out)
    return o, lse, m, dq, dk, dv


@pytest.mark.parametrize("mode", ["dense", "sparse", "causal"])
def test_outputs_and_workspace_stay_inside_their_buffers(mode):
    import torch
    L_k = 200 if mode == "causal" else 300
    w = W.custom(1, 2, 200, L_k, 128, seed_index=960)
    inp = W.inputs(w)
    q, k, v, dO = (to_gpu_bf16(inp[n]) for n in ("q", "k", "v", "do"))
    dev = q.device
    flags = oracle.QUANT_ALL | (A.CAUSAL if mode == "causal" else 0)
    tm = None
    if mode == "sparse":
        mask = W.random_tile_mask(w, 0.5)
        mask[0, 0, 1, :] = 0
        mask[0, 1, -1, -1] = 1
        tm = torch.from_numpy(mask).to(dev)
        need = A.attnqat_sparse_workspace_size(w.B, w.H, w.Lq, w.Lk, w.D, flags)
    else:
        need = A.attnqat_workspace_size(w.B, w.H, w.Lq, w.Lk, w.D, flags)
    bufs, outs = [], []
    for shape, dtype in (((1, 2, 200, 128), torch.bfloat16), ((1, 2, 200), torch.float32),
                         ((1, 2, 200), torch.float32), ((1, 2, 200, 128), torch.bfloat16),
                         ((1, 2, L_k, 128), torch.bfloat16), ((1, 2, L_k, 128), torch.bfloat16)):
        b, t = guarded(shape, dtype, dev)
        bufs.append(b)
        outs.append(t)
    bws, ws = guarded((need,), torch.uint8, dev)
    _call(mode, q, k, v, dO, w.sm_scale, flags, tm, outs=tuple(outs), ws=ws)
    torch.cuda.synchronize()
    A.attnqat_device_status()
    for name, b in zip(("o", "lse", "m", "dq", "dk", "dv", "workspace"), bufs + [bws]):
        assert guards_intact(b), name
    ref = _call(mode, q, k, v, dO, w.sm_scale, flags, tm)
    torch.cuda.synchronize()
    for name, got, want in zip(("o", "lse", "m", "dq", "dk", "dv"), outs, ref):
        assert torch.equal(got, want), name
