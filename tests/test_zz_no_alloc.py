"""csa_attend_noalloc: attention for callers that cannot allocate device memory.

Some callers only hold a stream and their tensors -- a plugin inside another
runtime, a serving loop that must not call cudaMalloc (it synchronises the
device), or code being captured into a CUDA graph -- so they cannot provide
the split-KV scratch that csa_attend takes.  csa_attend_noalloc uses a fixed
device array inside the library instead.  This test calls it through the C ABI
twice in a row, on different inputs, and checks each result against
csa_attend with a caller workspace (same tolerance as the other attention
tests; the kernels are the same, so the results should also be bit-identical).
It lives in a file pytest collects last, and works both alone and after the
rest of the suite.
"""
import numpy as np
import pytest
import torch

from long_context_compressed_06_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(seed, batch=8, H=128, D=512, N=4096, k=1024, Wn=128, m=4):
    dev = "cuda"
    T = N * m
    q = W.normal_bf16((batch, 1, H, D), seed, dev)
    kv = W.normal_bf16((batch, N, D), seed + 1, dev)
    win = W.normal_bf16((batch, Wn, D), seed + 2, dev)
    g = torch.Generator(device="cpu").manual_seed(seed + 3)
    idx = torch.stack([torch.randperm(N, generator=g)[:k].sort().values for _ in range(batch)])
    idx = idx.view(batch, 1, k).to(torch.int32).to(dev)
    qp = torch.full((batch, 1), T - 1, dtype=torch.int32, device=dev)
    return q, kv, idx, win, qp, Wn, D ** -0.5, T - Wn


def test_attend_noalloc_matches_attend_on_two_calls(cuda):
    import long_context_compressed_06_b200 as csa
    for seed in (500, 600):   # two calls in a row: the shared scratch keeps the previous contents
        q, kv, idx, win, qp, Wn, scale, p0 = _case(seed)
        ref = csa.csa_attend(q, kv, idx, win, qp, Wn, scale, win_pos0=p0)
        got = csa.csa_attend_noalloc(q, kv, idx, win, qp, Wn, scale, win_pos0=p0)
        assert csa.csa_sync_status() == 0
        r, o = ref.float().cpu().numpy(), got.float().cpu().numpy()
        assert np.abs(o - r).max() <= 2e-2 * np.abs(r).max()
        assert torch.equal(ref, got)


def test_attend_noalloc_rejects_sizes_beyond_its_scratch(cuda):
    import long_context_compressed_06_b200 as csa
    # a decode batch whose split-KV scratch is larger than the library's array
    batch = next(b for b in range(1, 512)
                 if csa.attend_workspace_bytes(b, 1, 128, 512, 1024 + 128) > 32 * 1024 * 1024)
    q = torch.zeros((batch, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((batch, 64, 512), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((batch, 1, 1024), dtype=torch.int32, device="cuda")
    win = torch.zeros((batch, 128, 512), dtype=torch.bfloat16, device="cuda")
    qp = torch.full((batch, 1), 255, dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError) as e:
        csa.csa_attend_noalloc(q, kv, idx, win, qp, 128, 512 ** -0.5)
    assert e.value.status == csa.CSA_ERR_WORKSPACE
