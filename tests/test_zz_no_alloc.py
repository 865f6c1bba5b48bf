"""attnqat_fwd_noalloc: the forward for callers that cannot allocate device
memory (its workspace is a block the library itself carries).  Checked through
the C ABI against attnqat_fwd with a caller-provided workspace, on two calls
in a row, so that a stale block from the previous call cannot hide a fault.

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


def _noalloc_fwd(q, k, v, c, flags):
    import torch
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    m = torch.empty_like(lse)
    st = _lib().attnqat_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        B, H, Lq, Lk, D, c, flags, ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(m.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, o, lse, m


@pytest.mark.parametrize("flags", [15, 4 | 8])
def test_noalloc_forward_matches_workspace_forward_twice(flags):
    import torch
    import quantization_aware_attention_nvfp4_b200 as A
    w = W.custom(1, 2, 300, 336, 128, seed_index=900 + flags)
    inp = W.inputs(w, with_grad=False)
    q, k, v = (to_gpu_bf16(inp[n]) for n in ("q", "k", "v"))
    c = 1.0 / math.sqrt(128)
    assert A.attnqat_workspace_size(1, 2, 300, 336, 128, flags) <= (32 << 20)
    o_ref, lse_ref, m_ref, _ = A.attnqat_fwd(q, k, v, sm_scale=c, flags=flags)
    torch.cuda.synchronize()
    for _ in range(2):
        st, o, lse, m = _noalloc_fwd(q, k, v, c, flags)
        assert st == A.OK, A.load().attnqat_strerror(st)
        torch.cuda.synchronize()
        A.attnqat_device_status()
        assert_close("O", to_f64(o), to_f64(o_ref))
        assert_close("LSE", to_f64(lse), to_f64(lse_ref))
        assert_close("m", to_f64(m), to_f64(m_ref))


def test_noalloc_rejects_shapes_beyond_its_block():
    import torch
    import quantization_aware_attention_nvfp4_b200 as A
    B, H, L, D = 1, 8, 16384, 128  # needs far more than 32 MiB of workspace
    assert A.attnqat_workspace_size(B, H, L, L, D, 15) > (32 << 20)
    q = torch.zeros((B, H, L, D), dtype=torch.bfloat16, device="cuda")
    st, _, _, _ = _noalloc_fwd(q, q, q, 0.1, 15)
    assert st == A.ENOSPC
