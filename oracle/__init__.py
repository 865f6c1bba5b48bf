"""Float64 CPU oracle for NVFP4 fake-quantized (Attn-QAT) attention.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the smoke check and by
the CPU-baseline leg of the benchmark, never by the library itself.  The
arithmetic lives in ``oracle.c`` (plain float64 C, OpenMP over independent
rows); this module only compiles it and marshals numpy arrays.

The method as restated here (see the header of ``oracle.c`` for the page
citations and the readings taken where the pages are silent):

* fq: E2M1 values, 16-element blocks along the contraction axis, E4M3 block
  scale = amax/6, round-to-nearest-even, no global scale
  (vsqa-test-1.3b metadata.json, "attention.precision" and
  "linear_quantization.format").
* forward: S = fq(Q) fq(K)^T c; m = row max; P~ = exp(S - m); l = sum P~;
  O = fq(P~) fq(V) / l; LSE = m + ln l.
* backward (straight-through): dV = (fq(P~)/l)^T dO; dS = P o (dO fq(V)^T -
  rowsum(dO o O)); dQ = dS fq(K) c; dK = dS^T fq(Q) c.
* block-sparse fine attention (vsqa-test-1.3b metadata.json, "attention":
  VSA_QAT_TRAIN_C128, 128-token cubes, selected key blocks per query block):
  the same computation restricted, per query tile, to the keys of the
  selected key tiles (``sel`` [n_query_tiles, n_key_tiles], nonzero =
  selected); a row with no selected key gives O = 0, LSE = m = -inf, dQ = 0.
* causal masking (flag CAUSAL, Lq == Lk): query i attends to keys j <= i.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against brute force, closed forms, torch's own float8 conversion and finite
differences; none is "parity unpinned".
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

QUANT_Q = 1
QUANT_K = 2
QUANT_V = 4
QUANT_P = 8
QUANT_ALL = 15
DV_QUANT_NORMALIZED = 16
CAUSAL = 32

_lock = threading.Lock()
_lib = None


def compile_library(src: str, out: str) -> str:
    """gcc (OpenMP, no floating-point contraction) of one oracle source file
    into a shared library at `out`."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
           "-std=c11", "-Wall", src, "-o", out, "-lm"]
    subprocess.check_call(cmd)
    return out


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP).  Returns the path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    compile_library(SRC, tmp)
    os.replace(tmp, LIB)
    return LIB


@contextlib.contextmanager
def library(path: str):
    """Test hook for the planted-mistake checks: inside the block every call of
    this module goes through the library at `path` (a build of a modified
    oracle.c); the previous library is restored on exit."""
    global _lib
    lib = _open(path)
    with _lock:
        saved, _lib = _lib, lib
    try:
        yield
    finally:
        with _lock:
            _lib = saved


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(build())
    return _lib


def _open(path: str):
    """The library at `path` with the argument types of its entry points."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    L = ctypes.c_long
    lib.oracle_bf16_value.restype = ctypes.c_double
    lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
    lib.oracle_e4m3_value.restype = ctypes.c_double
    lib.oracle_e4m3_value.argtypes = [ctypes.c_int]
    lib.oracle_e2m1_value.restype = ctypes.c_double
    lib.oracle_e2m1_value.argtypes = [ctypes.c_int]
    lib.oracle_e4m3_round_div6.restype = ctypes.c_int
    lib.oracle_e4m3_round_div6.argtypes = [ctypes.c_double]
    lib.oracle_e2m1_round.restype = ctypes.c_int
    lib.oracle_e2m1_round.argtypes = [ctypes.c_double, ctypes.c_double]
    lib.oracle_e2m1_round_many.restype = None
    lib.oracle_e2m1_round_many.argtypes = [P, P, L, P]
    lib.oracle_quantize_rows.restype = None
    lib.oracle_quantize_rows.argtypes = [P, L, L, L, L, P, P, P]
    lib.oracle_global_scale.restype = ctypes.c_float
    lib.oracle_global_scale.argtypes = [ctypes.c_double]
    lib.oracle_quantize_rows_gs.restype = None
    lib.oracle_quantize_rows_gs.argtypes = [P, L, L, L, L, P, P, P, P]
    lib.oracle_fq_f64_rows.restype = None
    lib.oracle_fq_f64_rows.argtypes = [P, L, L, P, P]
    lib.oracle_operands.restype = None
    lib.oracle_operands.argtypes = [P, P, P, L, L, L, ctypes.c_uint, P, P, P]
    lib.oracle_fwd_rows.restype = None
    lib.oracle_fwd_rows.argtypes = [P, P, P, L, L, L, ctypes.c_double,
                                    ctypes.c_uint, P, L, P, L, P, P, P, P]
    lib.oracle_delta.restype = None
    lib.oracle_delta.argtypes = [P, P, L, L, P]
    lib.oracle_bwd_dq_rows.restype = None
    lib.oracle_bwd_dq_rows.argtypes = [P, P, P, P, L, L, L, ctypes.c_double,
                                       ctypes.c_uint, P, L, P, P, P, P, L, P]
    lib.oracle_bwd_dkdv_blocks.restype = None
    lib.oracle_bwd_dkdv_blocks.argtypes = [P, P, P, P, L, L, L, ctypes.c_double,
                                           ctypes.c_uint, P, L, P, P, P, P, L, P, P]
    lib.oracle_vsa_select.restype = None
    lib.oracle_vsa_select.argtypes = [P, P, L, L, L, L, L, P, P]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 input as a contiguous uint16 numpy array of its bit patterns."""
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16), got %s" % a.dtype)
    return a


def num_threads() -> int:
    return _load().oracle_num_threads()


# ---------------------------------------------------------------- formats --

def bf16_value(bits: int) -> float:
    return _load().oracle_bf16_value(bits)


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(code)


def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(code)


def e4m3_round_div6(a: float) -> int:
    """Scale code: the nearest finite E4M3 to a/6, ties to even, saturating."""
    return _load().oracle_e4m3_round_div6(float(a))


def e2m1_round(ax: float, s: float) -> int:
    """Magnitude code: the nearest E2M1 value to ax/s, ties to even, saturating."""
    return _load().oracle_e2m1_round(float(ax), float(s))


def e2m1_round_many(ax: np.ndarray, s: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(ax, dtype=np.float64)
    b = np.ascontiguousarray(np.broadcast_to(s, a.shape), dtype=np.float64)
    out = np.zeros(a.shape, np.int32)
    _load().oracle_e2m1_round_many(_ptr(a), _ptr(b), a.size, _ptr(out))
    return out


# -------------------------------------------------------------- quantizer --

def quantize_rows(x_bits: np.ndarray, rows: int, cols: int, stride_row: int,
                  stride_col: int):
    """fq of each logical row of a strided bf16 view, blocks of 16 along cols.

    Returns (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16],
    deq float64 [rows, cols])."""
    x = _bits(x_bits).reshape(-1)
    if cols % 16:
        raise ValueError("cols must be a multiple of 16")
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    deq = np.zeros((rows, cols), np.float64)
    _load().oracle_quantize_rows(_ptr(x), rows, cols, stride_row, stride_col,
                                 _ptr(codes), _ptr(scales), _ptr(deq))
    return codes, scales, deq


def global_scale(amax: float) -> float:
    """The float32 global scale 2688 / amax (1 for amax = 0)."""
    return float(_load().oracle_global_scale(float(amax)))


def quantize_rows_gs(x_bits: np.ndarray, rows: int, cols: int, stride_row: int,
                     stride_col: int):
    """NVFP4 with an FP32 global scale of a strided bf16 view: G = float32
    2688 / max|x| (1 for an all-zero view), block scale = E4M3 of the exact
    a_b G / 6, code = E2M1 of the exact |x| G / s_b, value = sign * E2M1 *
    s_b / G rounded once to bf16 (the page gives the format, not the order of
    these steps; exact two-level rounding is the plain reading).

    Returns (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16],
    deq bf16 bits uint16 [rows, cols], global scale float)."""
    x = _bits(x_bits).reshape(-1)
    if cols % 16:
        raise ValueError("cols must be a multiple of 16")
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    deq = np.zeros((rows, cols), np.uint16)
    g = np.zeros(1, np.float32)
    _load().oracle_quantize_rows_gs(_ptr(x), rows, cols, stride_row, stride_col, _ptr(codes), _ptr(scales),
                                    _ptr(deq), _ptr(g))
    return codes, scales, deq, float(g[0])


def fq_f64_rows(x: np.ndarray):
    """fq of float64 rows in blocks of 16 (ragged last block zero-padded).
    Returns (dequantized float64, scale codes)."""
    a = np.ascontiguousarray(x, dtype=np.float64)
    rows, cols = a.shape
    y = np.zeros_like(a)
    sc = np.zeros((rows, (cols + 15) // 16), np.uint8)
    _load().oracle_fq_f64_rows(_ptr(a), rows, cols, _ptr(y), _ptr(sc))
    return y, sc


# -------------------------------------------------------------- attention --

class Head:
    """The fq'd float64 operands of one (b, h) head plus its dO.

    ``sel`` (optional, uint8 [ceil(Lq/tile), ceil(Lk/tile)]) restricts each
    query tile to the keys of its selected key tiles (block-sparse fine
    attention); ``tile`` is the tile length in tokens, a multiple of 16."""

    def __init__(self, q_bits, k_bits, v_bits, sm_scale, flags, do_bits=None, sel=None, tile=128):
        q = _bits(q_bits)
        k = _bits(k_bits)
        v = _bits(v_bits)
        self.Lq, self.D = q.shape
        self.Lk = k.shape[0]
        if v.shape != k.shape or k.shape[1] != self.D:
            raise ValueError("q [Lq,D], k and v [Lk,D] expected")
        if (flags & CAUSAL) and self.Lq != self.Lk:
            raise ValueError("causal masking needs Lq == Lk")
        if tile < 16 or tile % 16:
            raise ValueError("tile must be a positive multiple of 16")
        self.tile = int(tile)
        if sel is not None:
            sel = np.ascontiguousarray(sel, dtype=np.uint8)
            want = (-(-self.Lq // self.tile), -(-self.Lk // self.tile))
            if sel.shape != want:
                raise ValueError("sel must be [%d, %d]" % want)
        self.sel = sel
        self.c = float(sm_scale)
        self.flags = int(flags)
        self.Qh = np.zeros((self.Lq, self.D))
        self.Kh = np.zeros((self.Lk, self.D))
        self.Vh = np.zeros((self.Lk, self.D))
        _load().oracle_operands(_ptr(q), _ptr(k), _ptr(v), self.Lq, self.Lk, self.D,
                                self.flags, _ptr(self.Qh), _ptr(self.Kh), _ptr(self.Vh))
        self.dO = None if do_bits is None else _bits(do_bits)
        self._stats = None

    def _sel_ptr(self):
        return None if self.sel is None else _ptr(self.sel)

    # forward -------------------------------------------------------------
    def fwd_rows(self, rows=None):
        """O (float64), LSE, m, l for the listed query rows (all by default)."""
        rows = np.arange(self.Lq, dtype=np.int64) if rows is None else \
            np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        O = np.zeros((n, self.D))
        lse = np.zeros(n)
        m = np.zeros(n)
        l = np.zeros(n)
        _load().oracle_fwd_rows(_ptr(self.Qh), _ptr(self.Kh), _ptr(self.Vh), self.Lq,
                                self.Lk, self.D, self.c, self.flags, self._sel_ptr(), self.tile,
                                _ptr(rows), n, _ptr(O), _ptr(lse), _ptr(m), _ptr(l))
        return O, lse, m, l

    def stats(self):
        """Full-head forward statistics m, l, O and Delta = rowsum(dO o O)."""
        if self._stats is None:
            O, lse, m, l = self.fwd_rows()
            delta = np.zeros(self.Lq)
            if self.dO is not None:
                _load().oracle_delta(_ptr(O), _ptr(self.dO), self.Lq, self.D, _ptr(delta))
            self._stats = dict(O=O, lse=lse, m=m, l=l, delta=delta)
        return self._stats

    # backward ------------------------------------------------------------
    def dq_rows(self, rows=None):
        st = self.stats()
        rows = np.arange(self.Lq, dtype=np.int64) if rows is None else \
            np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        dQ = np.zeros((n, self.D))
        _load().oracle_bwd_dq_rows(_ptr(self.Qh), _ptr(self.Kh), _ptr(self.Vh),
                                   _ptr(self.dO), self.Lq, self.Lk, self.D, self.c,
                                   self.flags, self._sel_ptr(), self.tile, _ptr(st["m"]), _ptr(st["l"]),
                                   _ptr(st["delta"]), _ptr(rows), n, _ptr(dQ))
        return dQ

    def dkdv_blocks(self, blocks=None):
        """dK, dV for the keys of the listed 16-key blocks, [n*16, D] each
        (rows past Lk are zero)."""
        st = self.stats()
        nb = (self.Lk + 15) // 16
        blocks = np.arange(nb, dtype=np.int64) if blocks is None else \
            np.ascontiguousarray(blocks, dtype=np.int64)
        n = blocks.shape[0]
        dK = np.zeros((n * 16, self.D))
        dV = np.zeros((n * 16, self.D))
        _load().oracle_bwd_dkdv_blocks(_ptr(self.Qh), _ptr(self.Kh), _ptr(self.Vh),
                                       _ptr(self.dO), self.Lq, self.Lk, self.D, self.c,
                                       self.flags, self._sel_ptr(), self.tile, _ptr(st["m"]),
                                       _ptr(st["l"]),
                                       _ptr(st["delta"]), _ptr(blocks), n, _ptr(dK),
                                       _ptr(dV))
        return dK, dV

    def backward(self):
        """Full dQ, dK, dV of this head (float64)."""
        dQ = self.dq_rows()
        dK, dV = self.dkdv_blocks()
        return dQ, dK[: self.Lk], dV[: self.Lk]


def vsa_select(q_bits, k_bits, topk, tile=128):
    """Key-tile selection of block-sparse attention for one head: tile means,
    float32 coarse scores (mean query row . mean key row, every step in a
    fixed order, since the ranking decides an integer), the topk best key
    tiles per query tile (ties to the lower index).  q [Lq, D], k [Lk, D]
    bf16 bits.  Returns (mask uint8 [nq, nk], scores float32 [nq, nk])."""
    q = _bits(q_bits)
    k = _bits(k_bits)
    Lq, D = q.shape
    Lk = k.shape[0]
    if k.shape[1] != D or topk < 1 or tile < 1:
        raise ValueError("q [Lq,D], k [Lk,D], topk >= 1 expected")
    nq, nk = -(-Lq // tile), -(-Lk // tile)
    mask = np.zeros((nq, nk), np.uint8)
    scores = np.zeros((nq, nk), np.float32)
    _load().oracle_vsa_select(_ptr(q), _ptr(k), Lq, Lk, D, tile, int(topk), _ptr(mask), _ptr(scores))
    return mask, scores


def attention(q_bits, k_bits, v_bits, sm_scale, flags=QUANT_ALL, do_bits=None, sel=None, tile=128):
    """Full forward (and backward when dO is given) over [B, H, L, D] inputs;
    ``sel`` [B, H, n_query_tiles, n_key_tiles] makes it block-sparse.

    Returns a dict of float64 arrays: O, lse, m (and dQ, dK, dV)."""
    q = _bits(q_bits)
    k = _bits(k_bits)
    v = _bits(v_bits)
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    out = dict(O=np.zeros((B, H, Lq, D)), lse=np.zeros((B, H, Lq)), m=np.zeros((B, H, Lq)))
    if do_bits is not None:
        dO = _bits(do_bits)
        out.update(dQ=np.zeros((B, H, Lq, D)), dK=np.zeros((B, H, Lk, D)),
                   dV=np.zeros((B, H, Lk, D)))
    for b in range(B):
        for h in range(H):
            hd = Head(q[b, h], k[b, h], v[b, h], sm_scale, flags,
                      None if do_bits is None else dO[b, h],
                      None if sel is None else sel[b, h], tile)
            st = hd.stats()
            out["O"][b, h] = st["O"]
            out["lse"][b, h] = st["lse"]
            out["m"][b, h] = st["m"]
            if do_bits is not None:
                dQ, dK, dV = hd.backward()
                out["dQ"][b, h] = dQ
                out["dK"][b, h] = dK
                out["dV"][b, h] = dV
    return out
