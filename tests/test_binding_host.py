"""Host-side argument checks of the Python binding, on the CPU.

The C ABI receives bare pointers, so the binding is where caller-supplied
output tensors, workspaces and streams are checked against the call's shapes
and device before anything is launched.  Here the library is replaced by a
recorder (no GPU, no launch) and CPU tensors stand in for CUDA ones; a tensor
on the `meta` device plays a tensor on another device."""
import ctypes
from types import SimpleNamespace

import pytest
import torch

import quantization_aware_attention_nvfp4_b200 as A

B, H, LQ, LK, D = 1, 2, 40, 72, 64
CPU = torch.device("cpu")


class RecordingLib:
    """Stands in for libattnqat: workspace queries return a fixed size, every
    other entry point records its name and reports success."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name.endswith("workspace_size"):
            return lambda *args: 4096

        def call(*args):
            self.calls.append(name)
            return A.OK
        return call


def _bf16_any_device(name, t, ndim=None):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
        raise ValueError("%s must be bfloat16" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims" % (name, ndim))


@pytest.fixture
def lib(monkeypatch):
    rec = RecordingLib()
    monkeypatch.setattr(A, "load", lambda build_if_needed=True: rec)
    monkeypatch.setattr(A, "_require_bf16_cuda", _bf16_any_device)
    monkeypatch.setattr(A, "_stream_ptr", lambda stream=None, device=None: ctypes.c_void_p(0))
    return rec


def _qkv(Lq=LQ, Lk=LK):
    q = torch.zeros((B, H, Lq, D), dtype=torch.bfloat16)
    k = torch.zeros((B, H, Lk, D), dtype=torch.bfloat16)
    v = torch.zeros((B, H, Lk, D), dtype=torch.bfloat16)
    return q, k, v


def _stats(dtype=torch.float32, device=CPU):
    return torch.zeros((B, H, LQ), dtype=dtype, device=device)


def _mask(tile=128):
    return torch.ones((B, H, -(-LQ // tile), -(-LK // tile)), dtype=torch.uint8)


def test_forward_accepts_matching_buffers_and_rejects_others(lib):
    q, k, v = _qkv()
    ws = torch.empty(4096, dtype=torch.uint8)
    good = (torch.empty_like(q), _stats(), _stats())
    A.attnqat_fwd(q, k, v, ws=ws, out=good)
    A.attnqat_sparse_fwd(q, k, v, _mask(), ws=ws, out=good)
    assert lib.calls == ["attnqat_fwd", "attnqat_sparse_fwd"]
    bad_outputs = [
        (torch.empty((B, H, LQ + 1, D), dtype=torch.bfloat16), _stats(), _stats()),  # o one row too long
        (torch.empty_like(q, dtype=torch.float16), _stats(), _stats()),              # o not bf16
        (torch.empty_like(q), _stats(torch.float64), _stats()),                      # lse not float32
        (torch.empty_like(q), _stats(), torch.zeros((B, H, 2 * LQ))[..., ::2]),      # m not contiguous
        (torch.empty_like(q), _stats(device=torch.device("meta")), _stats()),        # lse on another device
    ]
    for out in bad_outputs:
        with pytest.raises(ValueError):
            A.attnqat_fwd(q, k, v, ws=ws, out=out)
        with pytest.raises(ValueError):
            A.attnqat_sparse_fwd(q, k, v, _mask(), ws=ws, out=out)
    with pytest.raises(ValueError):
        A.attnqat_fwd(q, k, v, ws=torch.empty(4096, dtype=torch.uint8, device="meta"))
    with pytest.raises(ValueError):
        A.attnqat_fwd(q, k, v, ws=torch.empty(8192, dtype=torch.uint8)[::2])
    assert lib.calls == ["attnqat_fwd", "attnqat_sparse_fwd"]  # nothing reached the library


def test_backward_checks_the_forward_results_and_its_outputs(lib):
    q, k, v = _qkv()
    dO = torch.zeros_like(q)
    ws = torch.empty(4096, dtype=torch.uint8)
    good = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    A.attnqat_bwd(q, k, v, _stats(), _stats(), dO, ws, out=good)
    A.attnqat_sparse_bwd(q, k, v, _stats(), _stats(), dO, ws, _mask(), out=good)
    assert lib.calls == ["attnqat_bwd", "attnqat_sparse_bwd"]
    bad_calls = [
        dict(lse=torch.zeros((B, H, LK))),                                        # lse shaped for the keys
        dict(m=_stats(torch.bfloat16)),                                           # m not float32
        dict(dO=torch.zeros((B, H, LK, D), dtype=torch.bfloat16)),                 # dO not shaped like q
        dict(ws=torch.empty(4096, dtype=torch.uint8, device="meta")),             # ws on another device
        dict(out=(torch.empty_like(q), torch.empty_like(q), torch.empty_like(v))),  # dk shaped like q
        dict(out=(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v, dtype=torch.float32))),
    ]
    for bad in bad_calls:
        kw = dict(lse=_stats(), m=_stats(), dO=dO, ws=ws, out=good)
        kw.update(bad)
        with pytest.raises(ValueError):
            A.attnqat_bwd(q, k, v, kw["lse"], kw["m"], kw["dO"], kw["ws"], out=kw["out"])
        with pytest.raises(ValueError):
            A.attnqat_sparse_bwd(q, k, v, kw["lse"], kw["m"], kw["dO"], kw["ws"], _mask(), out=kw["out"])
    assert lib.calls == ["attnqat_bwd", "attnqat_sparse_bwd"]


def test_inputs_must_share_one_device(lib):
    q, k, v = _qkv()
    k_elsewhere = torch.zeros((B, H, LK, D), dtype=torch.bfloat16, device="meta")
    with pytest.raises(ValueError):
        A.attnqat_fwd(q, k_elsewhere, v)
    with pytest.raises(ValueError):
        A.attnqat_fwd(q, k, k_elsewhere)
    with pytest.raises(ValueError):
        A.attnqat_vsa_select(q, k_elsewhere, topk=1)
    with pytest.raises(ValueError):
        A.attnqat_vsa_select(q, k, topk=1, ws=torch.empty(4096, dtype=torch.uint8, device="meta"))
    A.attnqat_vsa_select(q, k, topk=1)
    assert lib.calls == ["attnqat_vsa_select_tiles"]


def test_stream_must_belong_to_the_tensors_device():
    stream = SimpleNamespace(device=torch.device("meta"), cuda_stream=1234)
    with pytest.raises(ValueError):
        A._stream_ptr(stream, CPU)
    assert A._stream_ptr(stream, torch.device("meta")).value == 1234
