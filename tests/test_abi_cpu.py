"""C-ABI tests that need no GPU: the library loads, exports every function
include/csa.h declares, and rejects bad arguments on the host before any
launch (so these run in a container without a CUDA device)."""
import ctypes
import os
import re

import pytest

import long_context_compressed_06_b200 as csa
from long_context_compressed_06_b200 import build as csa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def lib():
    csa_build.build()
    return csa.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:csa|hca)_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_pipeline_calls():
    names = declared_functions()
    for n in ("csa_compress", "csa_compress_dynamic", "csa_index", "csa_index_fp4", "csa_quantize_fp4", "csa_topk", "csa_attend",
              "hca_attend", "csa_sync_status", "csa_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_strerror_and_version(lib):
    for code in (0, -1, -2, -3, -4, -5):
        assert csa.strerror(code)
    assert "unknown" in csa.strerror(17)
    assert lib.csa_version() >= 10000


NULL = None
A16 = ctypes.c_void_p(0x10000)      # a 16-byte aligned fake device address (never dereferenced)
A16b = ctypes.c_void_p(0x20000)
MIS = ctypes.c_void_p(0x10008)      # misaligned


def test_compress_validation(lib):
    f = lib.csa_compress
    assert f(NULL, A16, A16, 1, 64, 64, 4, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_INVALID
    assert f(MIS, A16, A16, 1, 64, 64, 4, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_INVALID
    assert f(A16, A16, A16, 1, 64, 60, 4, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_INVALID   # d % 8
    assert f(A16, A16, A16, 1, 3, 64, 4, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_INVALID    # T < m
    assert f(A16, A16, A16, 0, 64, 64, 4, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_INVALID   # batch
    assert f(A16, A16, A16, 1, 64, 64, 4, 1, NULL, -1.0, A16b, NULL) == csa.CSA_ERR_INVALID   # eps
    assert f(A16, A16, A16, 1, 4096, 2048, 4, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED
    assert f(A16, A16, A16, 1, 4096, 64, 512, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED
    # large m reads the logits as float4: 4-byte aligned logits are refused before any launch
    assert f(A16, A16, ctypes.c_void_p(0x10004), 1, 4096, 64, 128, 1, NULL, 1e-6, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED


def test_compress_dynamic_validation(lib):
    f = lib.csa_compress_dynamic
    # (A, B, Za, Zb, bias, batch, T, d, m, rms, gain, eps, i0, ni, out, n_out, stream)
    ok = dict(A=A16, B=A16, Za=A16, Zb=NULL, bias=A16, batch=1, T=64, d=64, m=4, rms=1, gain=NULL, eps=1e-6,
              i0=0, ni=16, out=A16b, n_out=16)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["A"], a["B"], a["Za"], a["Zb"], a["bias"], a["batch"], a["T"], a["d"], a["m"], a["rms"],
                 a["gain"], a["eps"], a["i0"], a["ni"], a["out"], a["n_out"], NULL)

    assert call(A=NULL) == csa.CSA_ERR_INVALID
    assert call(bias=NULL) == csa.CSA_ERR_INVALID
    assert call(Za=MIS) == csa.CSA_ERR_INVALID
    assert call(Zb=MIS) == csa.CSA_ERR_INVALID
    assert call(bias=MIS) == csa.CSA_ERR_INVALID
    assert call(gain=ctypes.c_void_p(0x10002)) == csa.CSA_ERR_INVALID
    assert call(d=60) == csa.CSA_ERR_INVALID                   # d % 8
    assert call(T=3) == csa.CSA_ERR_INVALID                    # T < m
    assert call(batch=0) == csa.CSA_ERR_INVALID
    assert call(eps=-1.0) == csa.CSA_ERR_INVALID
    assert call(i0=-1, ni=1) == csa.CSA_ERR_INVALID
    assert call(ni=-1) == csa.CSA_ERR_INVALID
    assert call(i0=10, ni=7) == csa.CSA_ERR_INVALID            # (i0 + ni) * m > T
    assert call(i0=0, ni=16, n_out=15) == csa.CSA_ERR_INVALID  # out too short
    assert call(T=4096, d=2056, ni=1, n_out=1) == csa.CSA_ERR_UNSUPPORTED
    big = 1 << 62                                                  # i0 + ni would overflow
    assert call(i0=big, ni=big, n_out=big) == csa.CSA_ERR_INVALID
    assert call(i0=big, ni=1, n_out=big) == csa.CSA_ERR_INVALID


def test_fp8_kv_validation(lib):
    f = lib.csa_quantize_fp8_kv
    assert f(NULL, 4, 512, A16b, A16, NULL) == csa.CSA_ERR_INVALID
    assert f(A16, 4, 512, MIS, A16, NULL) == csa.CSA_ERR_INVALID
    assert f(A16, 4, 512, A16b, NULL, NULL) == csa.CSA_ERR_INVALID
    assert f(A16, 4, 192, A16b, A16, NULL) == csa.CSA_ERR_INVALID     # d % 128
    assert f(A16, -1, 512, A16b, A16, NULL) == csa.CSA_ERR_INVALID
    g = lib.csa_attend_fp8kv
    # (q, g, sinks, rc, rs, rn, kv8, kv8e, N, idx, k, win8, win8e, p0, rows, W, pos, b, nq, H, D, scale, eps, out, ws, wsb, st)
    base = [A16, NULL, NULL, NULL, NULL, 0, A16, A16, 300, A16, 64, A16, A16, 0, 2048, 16, A16, 1, 1, 8, 512, 0.125,
            1e-6, A16b, NULL, 0, NULL]

    def call(**kw):
        a = list(base)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return g(*a)

    assert call(a6=MIS) == csa.CSA_ERR_INVALID          # codes misaligned
    assert call(a7=NULL) == csa.CSA_ERR_INVALID         # exponents missing
    assert call(a12=NULL) == csa.CSA_ERR_INVALID        # window exponents missing
    assert call(a20=64) == csa.CSA_ERR_UNSUPPORTED      # D = 64: no whole 128-channel block
    h = lib.hca_attend_fp8kv
    assert h(A16, NULL, NULL, NULL, NULL, 0, A16, A16, 300, 0, A16, A16, 0, 2048, 16, A16, 1, 1, 8, 512, 0.125, 1e-6,
             A16b, NULL, 0, NULL) == csa.CSA_ERR_INVALID    # m


def test_index_validation(lib):
    f = lib.csa_index
    ok = (A16, A16, A16, A16)
    assert f(NULL, A16, A16, A16, 1, 1, 100, 64, 128, 4, A16b, NULL) == csa.CSA_ERR_INVALID
    assert f(*ok, 1, 1, 100, 64, 120, 4, A16b, NULL) == csa.CSA_ERR_INVALID          # d_I % 16
    assert f(*ok, 1, 1, 0, 64, 128, 4, A16b, NULL) == csa.CSA_ERR_INVALID            # N
    assert f(*ok, 1, 1, 100, 64, 128, 0, A16b, NULL) == csa.CSA_ERR_INVALID          # m
    assert f(*ok, 1, 1, 100, 512, 128, 4, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED     # H_I
    assert f(*ok, 1, 1, 100, 64, 128, 4, MIS, NULL) == csa.CSA_ERR_INVALID
    # one implementation (the tensor-core kernel): other head dims are refused on the host
    assert f(*ok, 1, 1, 100, 8, 48, 4, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED        # d_I = 48
    assert f(*ok, 1, 1, 100, 8, 272, 4, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED       # d_I > 256
    g = lib.csa_index_fp4
    assert g(A16, NULL, A16, A16, A16, A16, 1, 1, 100, 64, 128, 4, A16b, NULL) == csa.CSA_ERR_INVALID
    assert g(A16, A16, A16, A16, A16, A16, 1, 1, 100, 4, 32, 4, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED  # d_I = 32
    odd = ctypes.c_void_p(0x10001)
    assert g(A16, A16, A16, A16, odd, A16, 1, 1, 100, 64, 128, 4, A16b, NULL) == csa.CSA_ERR_INVALID  # k4s
    assert g(A16, odd, A16, A16, A16, A16, 1, 1, 100, 64, 128, 4, A16b, NULL) == csa.CSA_ERR_INVALID  # q4s
    assert g(A16, ctypes.c_void_p(0x10002), A16, A16, A16, A16, 1, 1, 100, 64, 128, 4, A16b, NULL) == \
        csa.CSA_ERR_INVALID                                                                             # q4s % 4
    assert g(A16, A16, A16, A16, A16, A16, 1, 1, 100, 256, 128, 4, A16b, NULL) == csa.CSA_ERR_UNSUPPORTED  # H_I


def test_quantize_validation(lib):
    f = lib.csa_quantize_fp4
    assert f(A16, 10, 24, A16b, A16, NULL) == csa.CSA_ERR_INVALID   # d % 16
    assert f(A16, 0, 32, A16b, A16, NULL) == csa.CSA_ERR_INVALID
    assert f(MIS, 1, 32, A16b, A16, NULL) == csa.CSA_ERR_INVALID


def test_topk_validation(lib):
    f = lib.csa_topk
    assert f(A16, A16, 1, 1, 100, 4, 0, A16b, NULL, 0, NULL) == csa.CSA_ERR_INVALID       # k
    assert f(A16, A16, 1, 1, 100, 4, 9000, A16b, NULL, 0, NULL) == csa.CSA_ERR_UNSUPPORTED
    assert f(A16, A16, 1, 1, 1 << 20, 4, 64, A16b, NULL, 0, NULL) == csa.CSA_ERR_UNSUPPORTED
    assert lib.csa_topk_workspace_bytes(8, 1, 32768, 1024) == 0


def test_rescore_validation_and_workspace(lib):
    f = lib.csa_rescore_topk
    ws = ctypes.c_void_p(0x40000)          # 256-byte aligned
    need = lib.csa_rescore_workspace_bytes(4, 1, 4096, 1024, 128)
    assert need >= 4 * 4096 * 4 + 4 * 1024 * 4 + 4 * 4096 * 128 * 2
    args = (A16, A16, A16, A16, 4096, 4, 1, 262144, 64, 128, 1024, A16b)
    assert f(NULL, *args[1:], ws, need, NULL) == csa.CSA_ERR_INVALID                    # q_idx
    assert f(*args[:3], NULL, *args[4:], ws, need, NULL) == csa.CSA_ERR_INVALID        # cand
    assert f(*args[:10], 0, A16b, ws, need, NULL) == csa.CSA_ERR_INVALID               # k
    assert f(*args[:10], 9000, A16b, ws, need, NULL) == csa.CSA_ERR_UNSUPPORTED
    assert f(*args[:8], 256, 256, 1024, A16b, ws, need, NULL) == csa.CSA_ERR_UNSUPPORTED  # query + 2 stages > smem
    assert f(*args[:8], 8, 48, 1024, A16b, ws, need, NULL) == csa.CSA_ERR_UNSUPPORTED    # d_I = 48
    assert f(*args, ws, need - 1, NULL) == csa.CSA_ERR_WORKSPACE
    assert f(*args, ctypes.c_void_p(0x40010), need, NULL) == csa.CSA_ERR_WORKSPACE     # misaligned workspace
    assert f(*args, NULL, need, NULL) == csa.CSA_ERR_WORKSPACE


def test_attend_validation_and_workspace(lib):
    f = lib.csa_attend
    args = dict(q=A16, g=NULL, sk=NULL, rc=NULL, rs=NULL, rn=0, kv=A16, N=300, idx=A16, k=64, win=A16, p0=0, T=2048,
                W=16, pos=A16, b=1, nq=1, H=8, D=64, scale=0.125, eps=1e-6, out=A16b)

    def call(ws=NULL, wsb=0, **kw):
        a = dict(args, **kw)
        return f(a["q"], a["g"], a["sk"], a["rc"], a["rs"], a["rn"], a["kv"], a["N"], a["idx"], a["k"], a["win"],
                 a["p0"], a["T"], a["W"], a["pos"], a["b"], a["nq"], a["H"], a["D"], a["scale"], a["eps"], a["out"],
                 ws, wsb, NULL)

    assert call(q=NULL) == csa.CSA_ERR_INVALID
    assert call(sk=ctypes.c_void_p(0x10002)) == csa.CSA_ERR_INVALID    # sinks not 4-byte aligned
    assert call(rc=A16, rn=100) == csa.CSA_ERR_INVALID                 # rope cos without sin
    assert call(rs=A16, rn=100) == csa.CSA_ERR_INVALID                 # rope sin without cos
    assert call(rc=A16, rs=ctypes.c_void_p(0x10002), rn=100) == csa.CSA_ERR_INVALID
    assert call(rc=A16, rs=A16b, rn=0) == csa.CSA_ERR_INVALID          # empty tables
    assert call(W=0) == csa.CSA_ERR_INVALID
    assert call(p0=-1) == csa.CSA_ERR_INVALID
    assert call(T=0) == csa.CSA_ERR_INVALID
    assert call(D=96) == csa.CSA_ERR_UNSUPPORTED
    assert call(H=256) == csa.CSA_ERR_UNSUPPORTED
    need = lib.csa_attend_workspace_bytes(1, 1, 8, 64, 1024 + 16)
    assert need > 0   # a single query with 1040 keys is split over several CTAs
    assert call(ws=A16, wsb=need - 1, k=1024) == csa.CSA_ERR_WORKSPACE
    assert call(ws=MIS, wsb=need, k=1024) == csa.CSA_ERR_WORKSPACE
    h = lib.hca_attend
    assert h(A16, NULL, NULL, NULL, NULL, 0, A16, 300, 0, A16, 0, 2048, 16, A16, 1, 1, 8, 64, 0.125, 1e-6, A16b,
             NULL, 0, NULL) == csa.CSA_ERR_INVALID    # m


def test_attend_noalloc_checks_arguments_before_its_size_limit(lib):
    """The allocation-free entry point reports a bad argument as csa_attend
    does (its own size limit is checked only after the arguments).  Only
    invalid calls here: a valid one would launch."""
    f = lib.csa_attend_noalloc

    def call(q=A16, idx=A16, W=16, D=512, H=128, k=1024, out=A16b):
        return f(q, NULL, NULL, NULL, NULL, 0, A16, 1 << 16, idx, k, A16, 0, 1 << 18, W, A16, 8, 1,
                 H, D, 0.05, 1e-6, out, NULL)

    assert call(q=NULL) == csa.CSA_ERR_INVALID
    assert call(out=MIS) == csa.CSA_ERR_INVALID
    assert call(idx=ctypes.c_void_p(0x10002)) == csa.CSA_ERR_INVALID   # idx not 4-byte aligned
    assert call(k=-1) == csa.CSA_ERR_INVALID
    assert call(W=0) == csa.CSA_ERR_INVALID
    assert call(D=96) == csa.CSA_ERR_UNSUPPORTED
    assert call(H=256) == csa.CSA_ERR_UNSUPPORTED
    # workspace sizing is monotone in the key count and batch
    assert lib.csa_attend_workspace_bytes(8, 1, 128, 512, 1152) >= lib.csa_attend_workspace_bytes(1, 1, 128, 512, 1152)


def test_binding_refuses_host_tensors_and_has_no_fallback():
    """Every call takes CUDA tensors only: host tensors raise before anything is
    computed, so no step can silently run on the CPU."""
    import torch
    x = torch.zeros((1, 64, 64), dtype=torch.bfloat16)
    L = torch.zeros((8, 64), dtype=torch.float32)
    with pytest.raises(TypeError, match="CUDA tensor"):
        csa.csa_compress(x, x, L, 4)
    with pytest.raises(TypeError, match="CUDA tensor"):
        csa.csa_compress_dynamic(x, x, None, None, L, 4)
    with pytest.raises(TypeError, match="CUDA tensor"):
        csa.csa_index(torch.zeros((1, 1, 4, 32), dtype=torch.bfloat16), torch.zeros((1, 1, 4)),
                      torch.zeros((1, 16, 32), dtype=torch.bfloat16), torch.zeros((1, 1), dtype=torch.int32), 4)
    with pytest.raises(TypeError, match="CUDA tensor"):
        csa.csa_quantize_fp4(torch.zeros((4, 64), dtype=torch.bfloat16))


def test_missing_library_raises(monkeypatch, tmp_path):
    from long_context_compressed_06_b200 import binding
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="not built"):
        binding.load()


def test_decode_step_validates_every_argument_first(lib):
    """csa_decode_step refuses a bad argument of any of its three calls before
    launching anything (only invalid calls here: a valid one would launch)."""
    f = lib.csa_decode_step

    def call(q_idx=A16, k_idx=A16, H_I=64, d_I=128, m=4, k=1024, scores=A16b, idx=A16, q=A16, kv=A16, W=128,
             H=128, D=512, out=A16b, ws=NULL, wsb=0):
        return f(q_idx, A16, k_idx, H_I, d_I, m, k, scores, idx, q, NULL, NULL, NULL, NULL, 0, kv, 32768, A16, 0,
                 128, W, A16, 8, 1, H, D, 0.05, 1e-6, out, ws, wsb, NULL)

    assert call(q_idx=NULL) == csa.CSA_ERR_INVALID
    assert call(scores=MIS) == csa.CSA_ERR_INVALID
    assert call(idx=ctypes.c_void_p(0x10002)) == csa.CSA_ERR_INVALID
    assert call(d_I=120) == csa.CSA_ERR_INVALID
    assert call(m=0) == csa.CSA_ERR_INVALID
    assert call(k=0) == csa.CSA_ERR_INVALID
    assert call(d_I=48) == csa.CSA_ERR_UNSUPPORTED
    assert call(k=9000) == csa.CSA_ERR_UNSUPPORTED
    assert call(q=NULL) == csa.CSA_ERR_INVALID
    assert call(W=0) == csa.CSA_ERR_INVALID
    assert call(D=96) == csa.CSA_ERR_UNSUPPORTED
    assert call(H=256) == csa.CSA_ERR_UNSUPPORTED
    assert call() == csa.CSA_ERR_WORKSPACE        # 8 decode queries need split scratch
