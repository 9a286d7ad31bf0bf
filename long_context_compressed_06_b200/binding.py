"""Thin Python binding of libcsa.so (include/csa.h), same names as the C ABI.

Argument marshalling only: every step runs in the library's CUDA kernels.
Tensors are torch CUDA tensors (PyTorch supplies device memory and the current
stream); outputs are allocated here when not given.  If the shared library is
missing the first call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa.so")

CSA_OK, CSA_ERR_INVALID, CSA_ERR_UNSUPPORTED, CSA_ERR_CUDA, CSA_ERR_WORKSPACE, CSA_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5

_lib = None


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (where, strerror(status), status))


def load() -> ctypes.CDLL:
    """Load libcsa.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libcsa.so is not built (%s); run `python -m long_context_compressed_06_b200.build`"
                           % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
    sig = {
        "csa_strerror": ([i32], ctypes.c_char_p),
        "csa_version": ([], i32),
        "csa_compress": ([P, P, P, i32, i64, i32, i32, i32, P, f32, P, P], i32),
        "csa_quantize_fp8_kv": ([P, i64, i32, P, P, P], i32),
        "csa_attend_fp8kv": ([P, P, P, P, P, i64, P, P, i64, P, i32, P, P, i64, i64, i32, P, i32, i32, i32, i32, f32,
                              f32, P, P, sz, P], i32),
        "hca_attend_fp8kv": ([P, P, P, P, P, i64, P, P, i64, i32, P, P, i64, i64, i32, P, i32, i32, i32, i32, f32,
                              f32, P, P, sz, P], i32),
        "csa_compress_dynamic": ([P, P, P, P, P, i32, i64, i32, i32, i32, P, f32, i64, i64, P, i64, P], i32),
        "csa_index": ([P, P, P, P, i32, i32, i64, i32, i32, i32, P, P], i32),
        "csa_quantize_fp4": ([P, i64, i32, P, P, P], i32),
        "csa_index_fp4": ([P, P, P, P, P, P, i32, i32, i64, i32, i32, i32, P, P], i32),
        "csa_topk_workspace_bytes": ([i32, i32, i64, i32], sz),
        "csa_topk": ([P, P, i32, i32, i64, i32, i32, P, P, sz, P], i32),
        "csa_rescore_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
        "csa_rescore_topk": ([P, P, P, P, i32, i32, i32, i64, i32, i32, i32, P, P, sz, P], i32),
        "csa_attend_workspace_bytes": ([i32, i32, i32, i32, i64], sz),
        "csa_attend": ([P, P, P, P, P, i64, P, i64, P, i32, P, i64, i64, i32, P, i32, i32, i32, i32, f32, f32, P, P, sz, P],
                       i32),
        "hca_attend": ([P, P, P, P, P, i64, P, i64, i32, P, i64, i64, i32, P, i32, i32, i32, i32, f32, f32, P, P, sz, P], i32),
        "csa_decode_step": ([P, P, P, i32, i32, i32, i32, P, P, P, P, P, P, P, i64, P, i64, P, i64, i64, i32, P, i32, i32,
                             i32, i32, f32, f32, P, P, sz, P], i32),
        "csa_attend_noalloc": ([P, P, P, P, P, i64, P, i64, P, i32, P, i64, i64, i32, P, i32, i32, i32, i32, f32, f32, P, P],
                               i32),
        "csa_sync_status": ([P], i32),
        "csa_set_wait_budget_ns": ([ctypes.c_ulonglong], None),
        "csa_selftest_wait_timeout": ([P], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def strerror(status: int) -> str:
    return load().csa_strerror(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != CSA_OK:
        raise CsaError(rc, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, ndim: Optional[int] = None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    # every call launches on the current device: a tensor on another GPU would be
    # read through the wrong context
    if t.device.index != torch.cuda.current_device():
        raise ValueError("%s is on %s but the current device is cuda:%d (use torch.cuda.device(...))"
                         % (name, t.device, torch.cuda.current_device()))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got %s" % (name, ndim, tuple(t.shape)))
    return t


# --------------------------------------------------------------------------- ops
def csa_compress(A, B, logits, m: int, apply_rmsnorm: bool = True, gain=None, eps: float = 1e-6, out=None):
    """A, B [batch][T][d] bf16; logits [2m][d] fp32 -> compressed entries [batch][T//m][d] bf16."""
    L = load()
    _need(A, torch.bfloat16, "A", 3)
    _need(B, torch.bfloat16, "B", 3)
    _need(logits, torch.float32, "logits", 2)
    batch, T, d = A.shape
    if B.shape != A.shape or logits.shape != (2 * m, d):
        raise ValueError("shape mismatch")
    if gain is not None:
        _need(gain, torch.float32, "gain", 1)
    if out is None:
        out = torch.empty((batch, T // m, d), dtype=torch.bfloat16, device=A.device)
    _check(L.csa_compress(_p(A), _p(B), _p(logits), batch, T, d, m, int(bool(apply_rmsnorm)), _p(gain),
                          float(eps), _p(out), _stream()), "csa_compress")
    return out


def csa_compress_dynamic(A, B, Za, Zb, bias, m: int, apply_rmsnorm: bool = True, gain=None, eps: float = 1e-6,
                         i0: int = 0, ni=None, out=None):
    """Compressed entries [i0, i0+ni) with input-dependent weights.  A, B, Za, Zb [batch][T][d] bf16 (Za / Zb
    may be None), bias [2m][d] fp32 -> out [batch][n_out][d] bf16 with rows i0..i0+ni-1 written (default: all
    T//m entries into a new tensor; pass a cache as `out` to append entries)."""
    L = load()
    _need(A, torch.bfloat16, "A", 3)
    _need(B, torch.bfloat16, "B", 3)
    for z, name in ((Za, "Za"), (Zb, "Zb")):
        if z is not None:
            _need(z, torch.bfloat16, name, 3)
            if z.shape != A.shape:
                raise ValueError("shape mismatch: %s" % name)
    _need(bias, torch.float32, "bias", 2)
    batch, T, d = A.shape
    if B.shape != A.shape or bias.shape != (2 * m, d):
        raise ValueError("shape mismatch")
    if gain is not None:
        _need(gain, torch.float32, "gain", 1)
    if ni is None:
        ni = T // m - i0
    if out is None:
        out = torch.zeros((batch, T // m, d), dtype=torch.bfloat16, device=A.device)
    _need(out, torch.bfloat16, "out", 3)
    if out.shape[0] != batch or out.shape[2] != d:
        raise ValueError("shape mismatch: out")
    _check(L.csa_compress_dynamic(_p(A), _p(B), _p(Za), _p(Zb), _p(bias), batch, T, d, m,
                                  int(bool(apply_rmsnorm)), _p(gain), float(eps), int(i0), int(ni), _p(out),
                                  out.shape[1], _stream()), "csa_compress_dynamic")
    return out


def csa_index(q_idx, w, k_idx, q_pos, m: int, scores=None):
    """q_idx [b][nq][H_I][d_I] bf16, w [b][nq][H_I] fp32, k_idx [b][N][d_I] bf16 -> scores [b][nq][N] fp32."""
    L = load()
    _need(q_idx, torch.bfloat16, "q_idx", 4)
    _need(w, torch.float32, "w", 3)
    _need(k_idx, torch.bfloat16, "k_idx", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H_I, d_I = q_idx.shape
    N = k_idx.shape[1]
    if scores is None:
        scores = torch.empty((batch, nq, N), dtype=torch.float32, device=q_idx.device)
    _check(L.csa_index(_p(q_idx), _p(w), _p(k_idx), _p(q_pos), batch, nq, N, H_I, d_I, m, _p(scores),
                       _stream()), "csa_index")
    return scores


def csa_quantize_fp4(x, packed=None, scales=None):
    """x [..., d] bf16 -> (packed [..., d/2] u8, scales [..., d/16] u8 e4m3)."""
    L = load()
    _need(x, torch.bfloat16, "x")
    d = x.shape[-1]
    rows = x.numel() // d
    if packed is None:
        packed = torch.empty(x.shape[:-1] + (d // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1] + (d // 16,), dtype=torch.uint8, device=x.device)
    _check(L.csa_quantize_fp4(_p(x), rows, d, _p(packed), _p(scales), _stream()), "csa_quantize_fp4")
    return packed, scales


def csa_index_fp4(q4, q4s, w, k4, k4s, q_pos, m: int, scores=None):
    L = load()
    for t, n in ((q4, "q4"), (q4s, "q4s"), (k4, "k4"), (k4s, "k4s")):
        _need(t, torch.uint8, n)
    _need(w, torch.float32, "w", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H_I, half = q4.shape
    N = k4.shape[1]
    if scores is None:
        scores = torch.empty((batch, nq, N), dtype=torch.float32, device=q4.device)
    _check(L.csa_index_fp4(_p(q4), _p(q4s), _p(w), _p(k4), _p(k4s), _p(q_pos), batch, nq, N, H_I, half * 2, m,
                           _p(scores), _stream()), "csa_index_fp4")
    return scores


def csa_topk(scores, q_pos, m: int, k: int, idx=None):
    """scores [b][nq][N] fp32 -> idx [b][nq][k] int32 (ascending, -1 padded)."""
    L = load()
    _need(scores, torch.float32, "scores", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, N = scores.shape
    if idx is None:
        idx = torch.empty((batch, nq, k), dtype=torch.int32, device=scores.device)
    _check(L.csa_topk(_p(scores), _p(q_pos), batch, nq, N, m, k, _p(idx), None, 0, _stream()), "csa_topk")
    return idx


def rescore_workspace_bytes(batch: int, nq: int, kc: int, k: int, d_I: int) -> int:
    return int(load().csa_rescore_workspace_bytes(batch, nq, kc, k, d_I))


def csa_rescore_topk(q_idx, w, k_idx, cand, k: int, idx=None, workspace=None):
    """Re-rank FP4 candidates cand [b][nq][kc] with the bf16 index keys; -> idx [b][nq][k]."""
    L = load()
    _need(q_idx, torch.bfloat16, "q_idx", 4)
    _need(w, torch.float32, "w", 3)
    _need(k_idx, torch.bfloat16, "k_idx", 3)
    _need(cand, torch.int32, "cand", 3)
    batch, nq, H_I, d_I = q_idx.shape
    N = k_idx.shape[1]
    kc = cand.shape[2]
    if idx is None:
        idx = torch.empty((batch, nq, k), dtype=torch.int32, device=q_idx.device)
    nbytes = rescore_workspace_bytes(batch, nq, kc, k, d_I)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q_idx.device)
    _check(L.csa_rescore_topk(_p(q_idx), _p(w), _p(k_idx), _p(cand), kc, batch, nq, N, H_I, d_I, k, _p(idx),
                              _p(workspace), workspace.numel() * workspace.element_size(), _stream()),
           "csa_rescore_topk")
    return idx


def attend_workspace_bytes(batch: int, nq: int, H: int, D: int, max_keys: int) -> int:
    return int(load().csa_attend_workspace_bytes(batch, nq, H, D, max_keys))


def _workspace(nbytes: int, device, workspace):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def _sinks(sinks, H):
    if sinks is not None:
        _need(sinks, torch.float32, "sinks", 1)
        if sinks.shape[0] != H:
            raise ValueError("sinks must hold one logit per head (%d), got %d" % (H, sinks.shape[0]))
    return _p(sinks)


def _rope(rope, D):
    """rope = (cos, sin) fp32 tables [positions][32] or None -> (cos ptr, sin ptr, positions)."""
    if rope is None:
        return None, None, 0
    cos, sin = rope
    _need(cos, torch.float32, "rope cos", 2)
    _need(sin, torch.float32, "rope sin", 2)
    if cos.shape != sin.shape or cos.shape[1] != 32 or D < 64:
        raise ValueError("rope tables must be [positions][32] (64 rotated channels, D >= 64)")
    return _p(cos), _p(sin), cos.shape[0]


def csa_attend(q, kv, idx, win, q_pos, W: int, scale: float, eps: float = 1e-6, q_gain=None, out=None,
               workspace=None, win_pos0: int = 0, sinks=None, rope=None):
    """q [b][nq][H][D], kv [b][N][D], idx [b][nq][k], win [b][rows][D] (bf16, stream-A rows of positions
    win_pos0..) -> out [b][nq][H][D] bf16.  sinks: optional per-head sink logits [H] fp32.  rope: optional
    (cos, sin) [positions][32] fp32 tables for partial RoPE (keys and window rows arrive rotated)."""
    L = load()
    _need(q, torch.bfloat16, "q", 4)
    _need(kv, torch.bfloat16, "kv", 3)
    _need(idx, torch.int32, "idx", 3)
    _need(win, torch.bfloat16, "win", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H, D = q.shape
    N, rows, k = kv.shape[1], win.shape[1], idx.shape[2]
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = _workspace(attend_workspace_bytes(batch, nq, H, D, k + W), q.device, workspace)
    _check(L.csa_attend(_p(q), _p(q_gain), _sinks(sinks, H), *_rope(rope, D), _p(kv), N, _p(idx), k, _p(win), int(win_pos0), rows, W,
                        _p(q_pos),
                        batch, nq, H, D, float(scale), float(eps), _p(out), _p(ws), wsb, _stream()), "csa_attend")
    return out


def csa_decode_step(q_idx, w, k_idx, q, kv, win, q_pos, m: int, k: int, W: int, scale: float, eps: float = 1e-6,
                    q_gain=None, scores=None, idx=None, out=None, workspace=None, win_pos0: int = 0, sinks=None,
                    rope=None):
    """csa_index -> csa_topk -> csa_attend as one call (the top-k and attention kernels launched as
    programmatic dependents of their predecessor); returns (scores, idx, out)."""
    L = load()
    _need(q_idx, torch.bfloat16, "q_idx", 4)
    _need(w, torch.float32, "w", 3)
    _need(k_idx, torch.bfloat16, "k_idx", 3)
    _need(q, torch.bfloat16, "q", 4)
    _need(kv, torch.bfloat16, "kv", 3)
    _need(win, torch.bfloat16, "win", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H_I, d_I = q_idx.shape
    H, D = q.shape[2], q.shape[3]
    N, rows = k_idx.shape[1], win.shape[1]
    if kv.shape[1] != N:
        raise ValueError("kv and k_idx must hold the same number of entries")
    if scores is None:
        scores = torch.empty((batch, nq, N), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((batch, nq, k), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = _workspace(attend_workspace_bytes(batch, nq, H, D, k + W), q.device, workspace)
    _check(L.csa_decode_step(_p(q_idx), _p(w), _p(k_idx), H_I, d_I, m, k, _p(scores), _p(idx), _p(q), _p(q_gain),
                             _sinks(sinks, H), *_rope(rope, D), _p(kv), N, _p(win), int(win_pos0), rows, W, _p(q_pos),
                             batch, nq, H, D, float(scale), float(eps), _p(out), _p(ws), wsb, _stream()),
           "csa_decode_step")
    return scores, idx, out


def hca_attend(q, kv, m: int, win, q_pos, W: int, scale: float, eps: float = 1e-6, q_gain=None, out=None,
               workspace=None, win_pos0: int = 0, sinks=None, rope=None):
    """Dense attention over every visible entry of kv [b][N][D] plus the window."""
    L = load()
    _need(q, torch.bfloat16, "q", 4)
    _need(kv, torch.bfloat16, "kv", 3)
    _need(win, torch.bfloat16, "win", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H, D = q.shape
    N, rows = kv.shape[1], win.shape[1]
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = _workspace(attend_workspace_bytes(batch, nq, H, D, N + W), q.device, workspace)
    _check(L.hca_attend(_p(q), _p(q_gain), _sinks(sinks, H), *_rope(rope, D), _p(kv), N, m, _p(win), int(win_pos0), rows, W, _p(q_pos),
                        batch, nq, H,
                        D, float(scale), float(eps), _p(out), _p(ws), wsb, _stream()), "hca_attend")
    return out


def csa_quantize_fp8_kv(x, codes=None, exps=None):
    """KV rows x [..., d] bf16 (d % 128 == 0) -> (e4m3 codes [..., d] u8, UE8M0 exponents [..., d/128] u8)."""
    L = load()
    _need(x, torch.bfloat16, "x")
    d = x.shape[-1]
    rows = x.numel() // d
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if exps is None:
        exps = torch.empty(x.shape[:-1] + (d // 128,), dtype=torch.uint8, device=x.device)
    _need(codes, torch.uint8, "codes")
    _need(exps, torch.uint8, "exps")
    if codes.shape != x.shape or exps.numel() != rows * (d // 128):
        raise ValueError("shape mismatch")
    _check(L.csa_quantize_fp8_kv(_p(x), rows, d, _p(codes), _p(exps), _stream()), "csa_quantize_fp8_kv")
    return codes, exps


def _fp8_rows(codes, exps, name):
    _need(codes, torch.uint8, name, 3)
    _need(exps, torch.uint8, name + " exponents", 3)
    if exps.shape != codes.shape[:2] + (codes.shape[2] // 128,):
        raise ValueError("%s exponents must be [..][..][D/128]" % name)


def csa_attend_fp8kv(q, kv8, kv8_exp, idx, win8, win8_exp, q_pos, W: int, scale: float, eps: float = 1e-6,
                     q_gain=None, out=None, workspace=None, win_pos0: int = 0, sinks=None, rope=None):
    """csa_attend over an FP8 KV cache: kv8 [b][N][D] / win8 [b][rows][D] e4m3 codes with UE8M0 exponents
    [..][D/128] (from csa_quantize_fp8_kv)."""
    L = load()
    _need(q, torch.bfloat16, "q", 4)
    _fp8_rows(kv8, kv8_exp, "kv8")
    _fp8_rows(win8, win8_exp, "win8")
    _need(idx, torch.int32, "idx", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H, D = q.shape
    N, rows, k = kv8.shape[1], win8.shape[1], idx.shape[2]
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = _workspace(attend_workspace_bytes(batch, nq, H, D, k + W), q.device, workspace)
    _check(L.csa_attend_fp8kv(_p(q), _p(q_gain), _sinks(sinks, H), *_rope(rope, D), _p(kv8), _p(kv8_exp), N, _p(idx),
                              k, _p(win8), _p(win8_exp), int(win_pos0), rows, W, _p(q_pos), batch, nq, H, D,
                              float(scale), float(eps), _p(out), _p(ws), wsb, _stream()), "csa_attend_fp8kv")
    return out


def hca_attend_fp8kv(q, kv8, kv8_exp, m: int, win8, win8_exp, q_pos, W: int, scale: float, eps: float = 1e-6,
                     q_gain=None, out=None, workspace=None, win_pos0: int = 0, sinks=None, rope=None):
    """hca_attend over an FP8 KV cache."""
    L = load()
    _need(q, torch.bfloat16, "q", 4)
    _fp8_rows(kv8, kv8_exp, "kv8")
    _fp8_rows(win8, win8_exp, "win8")
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H, D = q.shape
    N, rows = kv8.shape[1], win8.shape[1]
    if out is None:
        out = torch.empty_like(q)
    ws, wsb = _workspace(attend_workspace_bytes(batch, nq, H, D, N + W), q.device, workspace)
    _check(L.hca_attend_fp8kv(_p(q), _p(q_gain), _sinks(sinks, H), *_rope(rope, D), _p(kv8), _p(kv8_exp), N, m,
                              _p(win8), _p(win8_exp), int(win_pos0), rows, W, _p(q_pos), batch, nq, H, D,
                              float(scale), float(eps), _p(out), _p(ws), wsb, _stream()), "hca_attend_fp8kv")
    return out


def csa_attend_noalloc(q, kv, idx, win, q_pos, W: int, scale: float, eps: float = 1e-6, q_gain=None, out=None,
                       win_pos0: int = 0, sinks=None, rope=None):
    """csa_attend without a caller workspace: the library's own fixed device
    scratch is used (for callers that cannot allocate; see include/csa.h)."""
    L = load()
    _need(q, torch.bfloat16, "q", 4)
    _need(kv, torch.bfloat16, "kv", 3)
    _need(idx, torch.int32, "idx", 3)
    _need(win, torch.bfloat16, "win", 3)
    _need(q_pos, torch.int32, "q_pos", 2)
    batch, nq, H, D = q.shape
    N, rows, k = kv.shape[1], win.shape[1], idx.shape[2]
    if out is None:
        out = torch.empty_like(q)
    _check(L.csa_attend_noalloc(_p(q), _p(q_gain), _sinks(sinks, H), *_rope(rope, D), _p(kv), N, _p(idx), k, _p(win), int(win_pos0),
                                rows, W,
                                _p(q_pos), batch, nq, H, D, float(scale), float(eps), _p(out), _stream()),
           "csa_attend_noalloc")
    return out


def csa_sync_status() -> int:
    return int(load().csa_sync_status(_stream()))


def csa_set_wait_budget_ns(ns: int) -> None:
    load().csa_set_wait_budget_ns(int(ns))


def csa_selftest_wait_timeout() -> None:
    _check(load().csa_selftest_wait_timeout(_stream()), "csa_selftest_wait_timeout")
