"""Float64 CPU oracle for the hybrid CSA/HCA attention step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it and share no code with it.

Every function takes numpy arrays holding the exact bit patterns the GPU path
consumes (bf16 as ``uint16``, FP4 as packed ``uint8``) and returns float64
results computed by the plain loops in ``csa_oracle.c``.  The definitions, the
pages they follow and the readings taken where the pages are silent are
documented there, function by function.
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


def lib():
    """Load (building first if needed) liboracle.so."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_longlong, ctypes.c_double
        L.orc_num_threads.restype = i32
        L.orc_set_num_threads.argtypes = [i32]
        L.orc_compress.argtypes = [P, P, P, i32, i64, i32, i32, i32, P, f64, i64, i64, P]
        L.orc_compress_dynamic.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, P, f64, i64, i64, P]
        L.orc_rmsnorm_bf16.argtypes = [P, i64, i32, f64, P, P]
        L.orc_n_visible.argtypes = [i64, i32, i64]
        L.orc_n_visible.restype = i64
        L.orc_index.argtypes = [P, P, P, P, i32, i32, i64, i32, i32, i32, P]
        L.orc_topk.argtypes = [P, P, i32, i32, i64, i32, i32, P]
        L.orc_attend.argtypes = [P, P, P, P, i64, P, i32, P, i64, i64, i32, P, i32, i32, i32, i32,
                                 f64, f64, i32, P, P, P]
        L.orc_hca_attend.argtypes = [P, P, P, P, i64, i32, P, i64, i64, i32, P, i32, i32, i32, i32,
                                     f64, f64, i32, P, P, P]
        L.orc_rope.argtypes = [P, i64, i32, i32, P, P, P, i32, P]
        L.orc_quantize_fp8_kv.argtypes = [P, i64, i32, i32, P, P]
        L.orc_dequantize_fp8_kv.argtypes = [P, P, i64, i32, i32, P]
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint]
        L.orc_e2m1_decode.restype = f64
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint]
        L.orc_e4m3_decode.restype = f64
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e2m1_encode.restype = ctypes.c_uint
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode.restype = ctypes.c_uint
        L.orc_quantize_fp4.argtypes = [P, i64, i32, P, P]
        L.orc_dequantize_fp4.argtypes = [P, P, i64, i32, P]
        L.orc_index_fp4.argtypes = [P, P, P, P, P, P, i32, i32, i64, i32, i32, i32, P]
        L.orc_index_fp4.restype = i32
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _opt(a, dtype):
    if a is None:
        return None, None
    return _c(a, dtype)


def num_threads() -> int:
    return lib().orc_num_threads()


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


def n_visible(t: int, m: int, N: int) -> int:
    return lib().orc_n_visible(int(t), int(m), int(N))


def compress(A, B, logits, m, apply_rmsnorm=True, gain=None, eps=1e-6, i0=0, ni=None):
    """Compressed entries [i0, i0+ni) of A,B [batch][T][d] (bf16 bits) -> float64 [batch][ni][d]."""
    A, pA = _c(A, np.uint16)
    B, pB = _c(B, np.uint16)
    batch, T, d = A.shape
    assert B.shape == A.shape
    L, pL = _c(logits, np.float32)
    assert L.shape == (2 * m, d)
    g, pg = _opt(gain, np.float32)
    N = T // m
    if ni is None:
        ni = N - i0
    assert 0 <= i0 and i0 + ni <= N
    out = np.empty((batch, ni, d), np.float64)
    lib().orc_compress(pA, pB, pL, batch, T, d, m, int(bool(apply_rmsnorm)), pg, float(eps),
                       int(i0), int(ni), out.ctypes.data_as(ctypes.c_void_p))
    return out


def compress_dynamic(A, B, Za, Zb, bias, m, apply_rmsnorm=True, gain=None, eps=1e-6, i0=0, ni=None):
    """Compressed entries [i0, i0+ni) with input-dependent weights: A, B, Za, Zb [batch][T][d] bf16 bits
    (Za / Zb may be None = 0), bias [2m][d] -> float64 [batch][ni][d]."""
    A, pA = _c(A, np.uint16)
    B, pB = _c(B, np.uint16)
    batch, T, d = A.shape
    assert B.shape == A.shape
    za, pza = _opt(Za, np.uint16)
    zb, pzb = _opt(Zb, np.uint16)
    assert za is None or za.shape == A.shape
    assert zb is None or zb.shape == A.shape
    L, pL = _c(bias, np.float32)
    assert L.shape == (2 * m, d)
    g, pg = _opt(gain, np.float32)
    N = T // m
    if ni is None:
        ni = N - i0
    assert 0 <= i0 and i0 + ni <= N
    out = np.empty((batch, ni, d), np.float64)
    lib().orc_compress_dynamic(pA, pB, pza, pzb, pL, batch, T, d, m, int(bool(apply_rmsnorm)), pg, float(eps),
                               int(i0), int(ni), out.ctypes.data_as(ctypes.c_void_p))
    return out


def rmsnorm(x, eps=1e-6, gain=None):
    """RMSNorm over the last axis of bf16 bits -> float64."""
    x, px = _c(x, np.uint16)
    d = x.shape[-1]
    g, pg = _opt(gain, np.float32)
    out = np.empty(x.shape, np.float64)
    lib().orc_rmsnorm_bf16(px, x.size // d, d, float(eps), pg, out.ctypes.data_as(ctypes.c_void_p))
    return out


def index(q_idx, w, k_idx, q_pos, m):
    """Indexer scores: q_idx [b][nq][H_I][d_I], w [b][nq][H_I], k_idx [b][N][d_I] -> [b][nq][N]."""
    q, pq = _c(q_idx, np.uint16)
    w, pw = _c(w, np.float32)
    k, pk = _c(k_idx, np.uint16)
    qp, pqp = _c(q_pos, np.int32)
    batch, nq, H_I, d_I = q.shape
    N = k.shape[1]
    assert k.shape == (batch, N, d_I) and w.shape == (batch, nq, H_I) and qp.shape == (batch, nq)
    out = np.empty((batch, nq, N), np.float64)
    lib().orc_index(pq, pw, pk, pqp, batch, nq, N, H_I, d_I, m, out.ctypes.data_as(ctypes.c_void_p))
    return out


def topk(scores, q_pos, m, k):
    """Top-k of [b][nq][N] scores among visible entries -> int32 [b][nq][k] (score desc, -1 pad)."""
    s, ps = _c(scores, np.float64)
    qp, pqp = _c(q_pos, np.int32)
    batch, nq, N = s.shape
    out = np.empty((batch, nq, k), np.int32)
    lib().orc_topk(ps, pqp, batch, nq, N, m, k, out.ctypes.data_as(ctypes.c_void_p))
    return out


def _rope_tables(rope, q_pos):
    """rope = (cos, sin) tables [positions][rope_dim/2] or None -> (rope_dim, arrays, pointers)."""
    if rope is None:
        return 0, (None, None), (None, None)
    c, pc = _c(rope[0], np.float32)
    s, ps = _c(rope[1], np.float32)
    assert c.ndim == 2 and c.shape == s.shape
    assert int(np.max(q_pos)) < c.shape[0] and int(np.min(q_pos)) >= 0
    return 2 * c.shape[1], (c, s), (pc, ps)


def rope(x, pos, cos, sin, inverse=False):
    """Partial RoPE of float64 rows x [..., width] at integer positions pos [...] with tables
    cos / sin [positions][rope_dim/2] (the trailing rope_dim channels rotate) -> float64."""
    x, px = _c(x, np.float64)
    width = x.shape[-1]
    p, pp = _c(np.broadcast_to(pos, x.shape[:-1]), np.int32)
    c, pc = _c(cos, np.float32)
    s, ps = _c(sin, np.float32)
    assert c.shape == s.shape and 2 * c.shape[1] <= width
    assert int(p.max()) < c.shape[0] and int(p.min()) >= 0
    out = np.empty(x.shape, np.float64)
    lib().orc_rope(px, x.size // width, width, 2 * c.shape[1], pp, pc, ps, int(bool(inverse)),
                   out.ctypes.data_as(ctypes.c_void_p))
    return out


def attend(q, kv, idx, win, q_pos, W, scale, eps=1e-6, q_gain=None, win_pos0=0, sinks=None, rope=None):
    """CSA attention: q [b][nq][H][D], kv [b][N][D], idx [b][nq][k], win [b][rows][D] holding stream-A
    positions win_pos0.. -> float64 [b][nq][H][D].  rope = (cos, sin) applies partial RoPE to the
    query heads and its conjugate to the outputs (keys arrive rotated)."""
    q, pq = _c(q, np.uint16)
    kv, pkv = _c(kv, np.uint16)
    idx, pidx = _c(idx, np.int32)
    win, pwin = _c(win, np.uint16)
    qp, pqp = _c(q_pos, np.int32)
    g, pg = _opt(q_gain, np.float32)
    batch, nq, H, D = q.shape
    N = kv.shape[1]
    k = idx.shape[2]
    rows = win.shape[1]
    out = np.empty(q.shape, np.float64)
    s_, ps_ = _opt(sinks, np.float32)
    rd, _keep, (pc, ps) = _rope_tables(rope, qp)
    lib().orc_attend(pq, pg, ps_, pkv, N, pidx, k, pwin, int(win_pos0), rows, W, pqp, batch, nq, H, D,
                     float(scale), float(eps), rd, pc, ps, out.ctypes.data_as(ctypes.c_void_p))
    return out


def hca_attend(q, kv, m, win, q_pos, W, scale, eps=1e-6, q_gain=None, win_pos0=0, sinks=None, rope=None):
    """HCA attention over all visible entries + window -> float64 [b][nq][H][D]."""
    q, pq = _c(q, np.uint16)
    kv, pkv = _c(kv, np.uint16)
    win, pwin = _c(win, np.uint16)
    qp, pqp = _c(q_pos, np.int32)
    g, pg = _opt(q_gain, np.float32)
    batch, nq, H, D = q.shape
    N = kv.shape[1]
    rows = win.shape[1]
    out = np.empty(q.shape, np.float64)
    s_, ps_ = _opt(sinks, np.float32)
    rd, _keep, (pc, ps) = _rope_tables(rope, qp)
    lib().orc_hca_attend(pq, pg, ps_, pkv, N, m, pwin, int(win_pos0), rows, W, pqp, batch, nq, H, D,
                         float(scale), float(eps), rd, pc, ps, out.ctypes.data_as(ctypes.c_void_p))
    return out


def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(code)


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(code)


def e2m1_encode(x: float) -> int:
    return lib().orc_e2m1_encode(x)


def e4m3_encode(x: float) -> int:
    return lib().orc_e4m3_encode(x)


def quantize_fp4(x):
    """[rows...][d] bf16 bits -> (packed u8 [...][d/2], scales u8 [...][d/16])."""
    x, px = _c(x, np.uint16)
    d = x.shape[-1]
    assert d % 16 == 0
    rows = x.size // d
    packed = np.empty(x.shape[:-1] + (d // 2,), np.uint8)
    scales = np.empty(x.shape[:-1] + (d // 16,), np.uint8)
    lib().orc_quantize_fp4(px, rows, d, packed.ctypes.data_as(ctypes.c_void_p),
                           scales.ctypes.data_as(ctypes.c_void_p))
    return packed, scales


def dequantize_fp4(packed, scales):
    p, pp = _c(packed, np.uint8)
    s, ps = _c(scales, np.uint8)
    d = p.shape[-1] * 2
    rows = p.size // (d // 2)
    out = np.empty(p.shape[:-1] + (d,), np.float64)
    lib().orc_dequantize_fp4(pp, ps, rows, d, out.ctypes.data_as(ctypes.c_void_p))
    return out


def quantize_fp8_kv(x, block=128):
    """KV rows [..., d] bf16 bits -> (e4m3 codes u8 [..., d], UE8M0 block exponents u8 [..., d/block])."""
    x, px = _c(x, np.uint16)
    d = x.shape[-1]
    assert d % block == 0
    rows = x.size // d
    codes = np.empty(x.shape, np.uint8)
    exps = np.empty(x.shape[:-1] + (d // block,), np.uint8)
    lib().orc_quantize_fp8_kv(px, rows, d, block, codes.ctypes.data_as(ctypes.c_void_p),
                              exps.ctypes.data_as(ctypes.c_void_p))
    return codes, exps


def dequantize_fp8_kv(codes, exps, block=128):
    """(codes [..., d], exponents [..., d/block]) -> float64 [..., d] (each value exactly a bf16 number)."""
    c, pc = _c(codes, np.uint8)
    e, pe = _c(exps, np.uint8)
    d = c.shape[-1]
    assert e.shape == c.shape[:-1] + (d // block,)
    out = np.empty(c.shape, np.float64)
    lib().orc_dequantize_fp8_kv(pc, pe, c.size // d, d, block, out.ctypes.data_as(ctypes.c_void_p))
    return out


def index_fp4(q4, q4s, w, k4, k4s, q_pos, m):
    """FP4 indexer scores (dequantised operands, float64) -> [b][nq][N]."""
    q4, pq4 = _c(q4, np.uint8)
    q4s, pq4s = _c(q4s, np.uint8)
    w, pw = _c(w, np.float32)
    k4, pk4 = _c(k4, np.uint8)
    k4s, pk4s = _c(k4s, np.uint8)
    qp, pqp = _c(q_pos, np.int32)
    batch, nq, H_I, half = q4.shape
    d_I = half * 2
    N = k4.shape[1]
    out = np.empty((batch, nq, N), np.float64)
    rc = lib().orc_index_fp4(pq4, pq4s, pw, pk4, pk4s, pqp, batch, nq, N, H_I, d_I, m,
                             out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("orc_index_fp4: unsupported d_I")
    return out


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
