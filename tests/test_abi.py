"""The C ABI on a machine without a GPU: the library builds and loads, exports
every symbol include/attnqat.h declares, and rejects bad arguments on the host
before touching the device.  No call here reaches a CUDA launch: every case
fails validation first (fake pointers are never dereferenced)."""
import ctypes
import math

import pytest

import quantization_aware_attention_nvfp4_b200 as A

FAKE = 0x10000  # 256-byte aligned, never dereferenced: validation fails first


def P(x):
    return ctypes.c_void_p(x)


def test_library_exports_every_declared_symbol():
    lib = A.load()
    names = A.header_symbols()
    assert {"attnqat_quantize", "attnqat_fwd", "attnqat_bwd", "attnqat_workspace_size",
            "attnqat_fwd_noalloc"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_strerror_texts():
    lib = A.load()
    for st in (A.OK, A.EINVAL, A.EUNSUPPORTED, A.ENOSPC, A.ECUDA, A.ETIMEOUT):
        assert lib.attnqat_strerror(st)
    assert lib.attnqat_strerror(-99) == b"unknown status"


def _expected_ws(B, H, Lq, Lk, D, flags):
    """Workspace layout restated: 256-byte aligned regions for the fp16
    copies of Q, K and V (fq or scaled), float32 O, Delta, 32 bytes of
    statistics, the fp16 copy of dO, with Q and K quantized their packed codes
    and scale tiles, and with every quantizer on and Lk % 32 == 0 fq(V)'s
    packed codes and scale tiles."""
    al = lambda x: (x + 255) // 256 * 256
    BH = B * H
    n = al(BH * Lq * D * 2) + 2 * al(BH * Lk * D * 2)
    n += al(BH * Lq * D * 4) + al(BH * Lq * 4) + al(32)
    n += al(BH * Lq * D * 2)  # fp16 copy of dO
    if flags & 3 == 3:
        # packed NVFP4 codes (D/2 bytes per row) and 512-byte scale tiles per
        # 128 rows x 64 columns, for Q then K
        for L in (Lq, Lk):
            n += al(BH * L * D // 2) + al(BH * ((L + 127) // 128) * (D // 64) * 512)
    if flags & 15 == 15 and Lk % 32 == 0:
        # fq(V)'s packed codes and 1 KB of scales per 128-token tile
        n += al(BH * Lk * D // 2) + al(BH * ((Lk + 127) // 128) * 1024)
    return n


@pytest.mark.parametrize("shape", [(1, 6, 31200, 31200, 128), (2, 3, 5, 48, 64), (1, 1, 1, 16, 128)])
@pytest.mark.parametrize("flags", [0, 15, 4, 3])
def test_workspace_size(shape, flags):
    assert A.attnqat_workspace_size(*shape, flags) == _expected_ws(*shape, flags)


@pytest.mark.parametrize("shape", [(0, 1, 16, 16, 128), (1, 1, 0, 16, 128), (1, 1, 16, 0, 128),
                                   (1, 1, 16, 16, 96), (1, 70000, 16, 16, 64)])
def test_workspace_size_rejects_bad_shapes(shape):
    assert A.attnqat_workspace_size(*shape, 15) == 0


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, B=1, H=1, Lq=128, Lk=128, D=128, c=0.125, flags=15, o=FAKE,
         lse=FAKE, m=FAKE, ws=FAKE, ws_bytes=0):
    return lib.attnqat_fwd(P(q), P(k), P(v), B, H, Lq, Lk, D, c, flags, P(o), P(lse), P(m), P(ws),
                           ws_bytes, None)


def test_fwd_host_validation():
    lib = A.load()
    big = 1 << 30
    assert _fwd(lib, q=0, ws_bytes=big) == A.EINVAL               # null input
    assert _fwd(lib, o=FAKE + 2, ws_bytes=big) == A.EINVAL        # misaligned output
    assert _fwd(lib, ws=FAKE + 16, ws_bytes=big) == A.EINVAL      # workspace not 256-byte aligned
    assert _fwd(lib, Lk=0, ws_bytes=big) == A.EINVAL             # no keys
    assert _fwd(lib, D=96, ws_bytes=big) == A.EUNSUPPORTED        # head dimension
    for c in (0.0, -1.0, math.inf, math.nan):                     # sm_scale used as given, must be valid
        assert _fwd(lib, c=c, ws_bytes=big) == A.EINVAL
    assert _fwd(lib, flags=16, ws_bytes=big) == A.EINVAL          # unknown flag bit
    assert _fwd(lib, ws_bytes=A.attnqat_workspace_size(1, 1, 128, 128, 128, 15) - 1) == A.ENOSPC


def test_bwd_host_validation():
    lib = A.load()
    big = 1 << 30

    def bwd(dO=FAKE, Lk=128, ws_bytes=big, c=0.125):
        return lib.attnqat_bwd(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(dO), 1, 1, 128, Lk, 128, c, 15,
                               P(FAKE), P(FAKE), P(FAKE), P(FAKE), ws_bytes, None)
    assert bwd(dO=0) == A.EINVAL
    assert bwd(Lk=0) == A.EINVAL
    assert bwd(c=math.nan) == A.EINVAL
    assert bwd(ws_bytes=16) == A.ENOSPC


def test_quantize_host_validation():
    lib = A.load()

    def quant(x=FAKE, batch=1, rows=4, cols=32, sb=0, sr=32, sc=1, codes=FAKE, scales=FAKE):
        return lib.attnqat_quantize(P(x), batch, rows, cols, sb, sr, sc, P(codes), P(scales), None, None)
    assert quant(x=0) == A.EINVAL
    assert quant(codes=0) == A.EINVAL
    assert quant(cols=24) == A.EINVAL
    assert quant(rows=0) == A.EINVAL
    assert quant(sr=-1) == A.EINVAL
    assert quant(x=FAKE + 1) == A.EINVAL
    assert quant(codes=FAKE + 4) == A.EINVAL  # codes are written as 8-byte groups


def test_noalloc_rejects_oversized_shapes_before_any_device_call():
    lib = A.load()
    lib.attnqat_fwd_noalloc.restype = ctypes.c_int
    lib.attnqat_fwd_noalloc.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + \
        [ctypes.c_float, ctypes.c_uint32] + [ctypes.c_void_p] * 4
    st = lib.attnqat_fwd_noalloc(P(FAKE), P(FAKE), P(FAKE), 1, 8, 16384, 16384, 128, 0.1, 15,
                                 P(FAKE), P(FAKE), P(FAKE), None)
    assert st == A.ENOSPC
    st = lib.attnqat_fwd_noalloc(P(FAKE), P(FAKE), P(FAKE), 1, 1, 16, 0, 128, 0.1, 15,
                                 P(FAKE), P(FAKE), P(FAKE), None)
    assert st == A.EINVAL


def test_python_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros((1, 1, 16, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        A.attnqat_fwd(x, x, x)


def test_quantize_gs_host_validation():
    lib = A.load()

    def quant(x=FAKE, cols=32, codes=FAKE, g=FAKE):
        return lib.attnqat_quantize_gs(P(x), 1, 4, cols, 0, cols, 1, P(codes), P(FAKE), None, P(g), None)
    assert quant(g=0) == A.EINVAL
    assert quant(g=FAKE + 2) == A.EINVAL     # float32 slot misaligned
    assert quant(x=0) == A.EINVAL
    assert quant(codes=0) == A.EINVAL
    assert quant(codes=FAKE + 4) == A.EINVAL
    assert quant(cols=24) == A.EINVAL


@pytest.mark.parametrize("shape", [(1, 6, 31200, 31200, 128), (2, 3, 5, 300, 64)])
def test_sparse_workspace_size(shape):
    """The dense workspace plus int32 tile lists: [BH][nq][nk] and [BH][nk][nq]
    with their counts, each region 256-byte aligned."""
    al = lambda x: (x + 255) // 256 * 256
    B, H, Lq, Lk, D = shape
    BH, nq, nk = B * H, -(-Lq // 128), -(-Lk // 128)
    extra = 2 * al(BH * nq * nk * 4) + al(BH * nq * 4) + al(BH * nk * 4)
    assert A.attnqat_sparse_workspace_size(*shape, 15) == _expected_ws(*shape, 15) + extra


def test_sparse_host_validation():
    lib = A.load()
    big = 1 << 30

    def fwd(mask=FAKE, q=FAKE, Lk=128, ws_bytes=big):
        return lib.attnqat_sparse_fwd(P(q), P(FAKE), P(FAKE), 1, 1, 128, Lk, 128, 0.125, 15, P(mask), P(FAKE),
                                      P(FAKE), P(FAKE), P(FAKE), ws_bytes, None)

    def bwd(mask=FAKE, ws_bytes=big):
        return lib.attnqat_sparse_bwd(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1, 1, 128, 128, 128,
                                      0.125, 15, P(mask), P(FAKE), P(FAKE), P(FAKE), P(FAKE), ws_bytes, None)
    assert fwd(mask=0) == A.EINVAL
    assert fwd(q=0) == A.EINVAL
    assert fwd(Lk=0) == A.EINVAL
    # the dense workspace is too small for the tile lists
    assert fwd(ws_bytes=A.attnqat_workspace_size(1, 1, 128, 128, 128, 15)) == A.ENOSPC
    assert bwd(mask=0) == A.EINVAL
    assert bwd(ws_bytes=A.attnqat_sparse_workspace_size(1, 1, 128, 128, 128, 15) - 1) == A.ENOSPC


def test_vsa_select_host_validation_and_workspace():
    lib = A.load()
    al = lambda x: (x + 255) // 256 * 256
    B, H, Lq, Lk, D = 1, 6, 31200, 31200, 128
    nq = nk = 244
    assert A.load().attnqat_vsa_select_workspace_size(B, H, Lq, Lk, D) == \
        al(B * H * (nq + nk) * D * 4) + al(B * H * nq * nk * 4)
    assert A.load().attnqat_vsa_select_workspace_size(1, 1, 16, 16, 96) == 0
    big = 1 << 30

    def sel(q=FAKE, topk=3, mask=FAKE, ws=FAKE, ws_bytes=big, D=128):
        return lib.attnqat_vsa_select(P(q), P(FAKE), 1, 1, 300, 700, D, topk, P(mask), P(ws), ws_bytes, None)
    assert sel(q=0) == A.EINVAL
    assert sel(mask=0) == A.EINVAL
    assert sel(topk=0) == A.EINVAL
    assert sel(ws=FAKE + 16) == A.EINVAL
    assert sel(D=96) == A.EUNSUPPORTED
    assert sel(ws_bytes=lib.attnqat_vsa_select_workspace_size(1, 1, 300, 700, 128) - 1) == A.ENOSPC


def test_causal_flag_validation_and_workspace():
    lib = A.load()
    big = 1 << 30
    # causal needs Lq == Lk
    assert _fwd(lib, Lq=128, Lk=256, flags=15 | A.CAUSAL, ws_bytes=big) == A.EINVAL
    assert A.attnqat_workspace_size(1, 1, 128, 256, 128, 15 | A.CAUSAL) == 0
    # the causal workspace adds the tile lists of the lower triangle
    assert A.attnqat_workspace_size(1, 6, 31200, 31200, 128, 15 | A.CAUSAL) == \
        A.attnqat_sparse_workspace_size(1, 6, 31200, 31200, 128, 15)
    assert A.attnqat_sparse_workspace_size(1, 1, 128, 128, 128, 15 | A.CAUSAL) == 0
    assert _fwd(lib, flags=15 | A.CAUSAL,
                ws_bytes=A.attnqat_workspace_size(1, 1, 128, 128, 128, 15 | A.CAUSAL) - 1) == A.ENOSPC
    # no combination with a tile selection
    st = lib.attnqat_sparse_fwd(P(FAKE), P(FAKE), P(FAKE), 1, 1, 128, 128, 128, 0.125, 15 | A.CAUSAL, P(FAKE),
                                P(FAKE), P(FAKE), P(FAKE), P(FAKE), big, None)
    assert st == A.EINVAL
    assert _fwd(lib, flags=64, ws_bytes=big) == A.EINVAL  # still an unknown bit
    # every flag set takes causal masking (every backward operand is fp16)
    for flags in range(16):
        need = A.attnqat_workspace_size(1, 1, 128, 128, 128, flags | A.CAUSAL)
        assert need > A.attnqat_workspace_size(1, 1, 128, 128, 128, flags) > 0
        assert _fwd(lib, flags=flags | A.CAUSAL, ws_bytes=need - 1) == A.ENOSPC


def test_selftest_wait_timeout_validation():
    lib = A.load()
    assert lib.attnqat_selftest_wait_timeout(1000000, None, None) == A.EINVAL       # no counter
    assert lib.attnqat_selftest_wait_timeout(1000000, P(FAKE + 2), None) == A.EINVAL  # misaligned
    assert lib.attnqat_selftest_wait_timeout(999, P(FAKE), None) == A.EINVAL         # limit too short
    assert lib.attnqat_selftest_wait_timeout(3 * 10**9, P(FAKE), None) == A.EINVAL   # above 2 s


def test_tile64_flag_validation():
    lib = A.load()
    big = 1 << 30
    # the 64-token profile keeps the 128-token tile lists: the same workspace
    for flags in (15, 0, 3):
        assert A.attnqat_sparse_workspace_size(1, 6, 31200, 31200, 128, flags | A.TILE64) == \
            A.attnqat_sparse_workspace_size(1, 6, 31200, 31200, 128, flags)
    # a mask-only flag: not for the dense calls, not with causal masking
    assert A.attnqat_workspace_size(1, 1, 128, 128, 128, 15 | A.TILE64) == 0
    assert _fwd(lib, flags=15 | A.TILE64, ws_bytes=big) == A.EINVAL
    assert A.attnqat_sparse_workspace_size(1, 1, 128, 128, 128, 15 | A.TILE64 | A.CAUSAL) == 0
    # the selection takes 64- or 128-token tiles
    assert lib.attnqat_vsa_select_tiles_workspace_size(1, 1, 300, 700, 128, 96) == 0
    assert lib.attnqat_vsa_select_tiles_workspace_size(1, 1, 300, 700, 128, 128) == \
        lib.attnqat_vsa_select_workspace_size(1, 1, 300, 700, 128)
    nq, nk = -(-300 // 64), -(-700 // 64)
    al = lambda x: (x + 255) // 256 * 256
    assert lib.attnqat_vsa_select_tiles_workspace_size(1, 1, 300, 700, 128, 64) == \
        al((nq + nk) * 128 * 4) + al(nq * nk * 4)
    st = lib.attnqat_vsa_select_tiles(P(FAKE), P(FAKE), 1, 1, 300, 700, 128, 96, 3, P(FAKE), P(FAKE), big, None)
    assert st == A.EINVAL
