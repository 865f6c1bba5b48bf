"""attnqat_fwd_noalloc: the forward for callers that cannot allocate device
memory (a framework whose caching allocator already holds nearly all of it,
code inside an allocator callback, a C host with no device allocator): its
workspace is a block the library itself carries.  Checked through the C ABI
against attnqat_fwd with a caller-provided workspace, bit for bit (the same
kernels run on the same inputs), over a sequence of calls whose shapes,
inputs and flag sets change from one call to the next, so that what one call
leaves in the shared block cannot hide a fault in the next (a partial last
tile reading stale scale tiles, statistics that were not cleared).

This file is named to be collected last: it must pass both on its own in a
fresh process and after every other test."""
import ctypes
import math

import numpy as np
import pytest

from quantization_aware_attention_nvfp4_b200 import workloads as W
from tests.helpers import assert_close, to_f64, to_gpu_bf16

pytestmark = pytest.mark.gpu


def _lib():
    import quantization_aware_attention_nvfp4_b200 as A
    lib = A.load()
    P, I, U32, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_float
    lib.attnqat_fwd_noalloc.restype = I
    lib.attnqat_fwd_noalloc.argtypes = [P, P, P, I, I, I, I, I, F, U32, P, P, P, P]
    return lib


def _noalloc_fwd(q, k, v, c, flags, D=None):
    import torch
    B, H, Lq, Dq = q.shape
    D = Dq if D is None else D
    Lk = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    m = torch.empty_like(lse)
    st = _lib().attnqat_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        B, H, Lq, Lk, D, c, flags, ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(m.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, o, lse, m


# (B, H, Lq, Lk, D, flags): whole tiles, then ragged tiles, then whole tiles
# again with other flags, so every call follows one with another shape
SEQUENCE = [
    (1, 2, 256, 512, 128, 15),      # whole query and key tiles, NVFP4 P V
    (1, 2, 300, 336, 128, 15),      # partial last tiles (Lk % 128 = 80)
    (2, 1, 130, 1000, 64, 15),      # D = 64, Lk % 16 != 0
    (1, 2, 300, 336, 128, 4 | 8),   # fp16 copies of unquantized Q and K
    (1, 2, 256, 512, 128, 15),      # back to the first shape
    (1, 1, 200, 200, 128, 15 | 32),  # causal
]


def test_noalloc_forward_matches_workspace_forward_bitwise():
    import torch
    import quantization_aware_attention_nvfp4_b200 as A
    for i, (B, H, Lq, Lk, D, flags) in enumerate(SEQUENCE):
        assert A.attnqat_workspace_size(B, H, Lq, Lk, D, flags) <= (32 << 20)
        w = W.custom(B, H, Lq, Lk, D, seed_index=900 + i)
        inp = W.inputs(w, with_grad=False)
        q, k, v = (to_gpu_bf16(inp[n]) for n in ("q", "k", "v"))
        c = 1.0 / math.sqrt(D)
        o_ref, lse_ref, m_ref, _ = A.attnqat_fwd(q, k, v, sm_scale=c, flags=flags)
        torch.cuda.synchronize()
        st, o, lse, m = _noalloc_fwd(q, k, v, c, flags)
        assert st == A.OK, A.load().attnqat_strerror(st)
        torch.cuda.synchronize()
        A.attnqat_device_status()
        what = "call %d %s" % (i, SEQUENCE[i])
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16)), what
        assert torch.equal(lse, lse_ref) and torch.equal(m, m_ref), what
        # within the parity tolerance as well (implied by the bitwise match)
        assert_close("O", to_f64(o), to_f64(o_ref))


def test_noalloc_rejects_shapes_beyond_its_block():
    import torch
    import quantization_aware_attention_nvfp4_b200 as A
    B, H, L, D = 1, 8, 16384, 128  # needs far more than 32 MiB of workspace
    assert A.attnqat_workspace_size(B, H, L, L, D, 15) > (32 << 20)
    q = torch.zeros((B, H, L, D), dtype=torch.bfloat16, device="cuda")
    st, _, _, _ = _noalloc_fwd(q, q, q, 0.1, 15)
    assert st == A.ENOSPC


def test_noalloc_reports_argument_errors_like_attnqat_fwd():
    import quantization_aware_attention_nvfp4_b200 as A
    q = _zeros(1, 1, 64, 64)
    assert _noalloc_fwd(q, q, q, 0.1, 15, D=96)[0] == A.EUNSUPPORTED  # head dimension
    assert _noalloc_fwd(q, q, q, -1.0, 15)[0] == A.EINVAL               # softmax scale
    assert _noalloc_fwd(q, q, q, 0.1, 64)[0] == A.EINVAL                # unknown flag bit


def _zeros(B, H, L, D):
    import torch
    return torch.zeros((B, H, L, D), dtype=torch.bfloat16, device="cuda")
