"""GPU parity at the five workloads' own shapes (the launch configurations the
benchmark times), against the float64 oracle on the same seeded input bits.

Where the oracle cannot finish a whole workload in seconds, it checks sampled
queries (the first and last positions always among them); the GPU still runs
the whole workload in one launch.

Acceptance rules ("DeepSeek v4", "Compressed Sparse Attention" -> "sparse
selection Lightning Indexer": the top-k selector over the index scores):
  * top-k: the GPU's csa_index -> csa_topk selection may differ from the
    oracle's top-k of its own float64 scores only in entries whose oracle score
    lies within 1e-4 * |s_k| of the k-th oracle score s_k;
  * attention: max|err| <= 2e-2 * max|out| against the oracle on the same
    (seeded or oracle-derived) selection;
  * FP4 indexer ("DeepSeek V4 paper full version is out, FP4 QAT details and
    stability tricks", FP4 activations on the indexer QK path): scores exact
    to the FP4 values (1e-5 * max|S|); the selection after FP4 over-selection
    (4k candidates) and the bf16 re-rank recalls >= 99 % of the oracle's top-k
    of the bf16-operand scores.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_06_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_band(sel, ref_scores, q_pos, m, k, N):
    """sel [..][k] GPU indices against float64 scores [..][N]: set difference
    only inside the 1e-4 relative band around the k-th oracle score."""
    for q in np.ndindex(ref_scores.shape[:-1]):
        nv = oracle.n_visible(int(q_pos[q]), m, N)
        g = sel[q]
        gset = set(g[g >= 0].tolist())
        assert len(gset) == len(g[g >= 0]) == min(k, nv), q
        assert np.sum(g == -1) == max(0, k - nv), q
        if nv <= k:
            assert gset == set(range(nv)), q
            continue
        s = ref_scores[q][:nv]
        oset = set(oracle.topk(ref_scores[q][None, None], np.array([[q_pos[q]]], np.int32), m, k)[0, 0].tolist())
        sk = np.sort(s)[::-1][k - 1]
        band = 1e-4 * abs(sk)
        for j in gset ^ oset:
            assert abs(s[j] - sk) <= band, (q, j, s[j], sk)


def recall(sel, ref_sel):
    """|sel ∩ ref| / |ref|, pooled over queries (ref without its -1 slots)."""
    hit = tot = 0
    for q in np.ndindex(ref_sel.shape[:-1]):
        r = set(ref_sel[q][ref_sel[q] >= 0].tolist())
        g = set(sel[q][sel[q] >= 0].tolist())
        hit += len(r & g)
        tot += len(r)
    return hit / tot


# ----------------------------------------------------------------------------- index -> top-k chain
@pytest.mark.parametrize("wl", [W.TINY, W.CSA_DECODE], ids=lambda w: w.name)
def test_index_topk_chain_in_band(cuda, wl):
    """The real decode chain, GPU index scores selected by the GPU top-k, at the
    tiny and the 128K decode workloads (every query checked)."""
    qI, w, kI = W.index_queries(wl, DEV), W.index_weights(wl, DEV), W.index_keys(wl, DEV)
    qp = wl.q_positions().to(DEV)
    S = cuda.csa_index(qI, w, kI, qp, wl.m)
    sel = cuda.csa_topk(S, qp, wl.m, wl.k).cpu().numpy()
    assert cuda.csa_sync_status() == 0
    ref = oracle.index(W.bits(qI), w.cpu().numpy(), W.bits(kI), qp.cpu().numpy(), wl.m)
    check_band(sel, ref, qp.cpu().numpy(), wl.m, wl.k, wl.N)


def _prefill_rows(nq, n=64, seed=7):
    r = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, 1, nq // 2, nq - 2, nq - 1], r.choice(nq, n - 5, replace=False)]))
    return rows


def test_index_topk_chain_prefill_sampled_rows(cuda):
    """The prefill chunk (4096 queries at positions 61440..65535 over 16384
    entries): one csa_index launch and one csa_topk launch over every query;
    64 sampled query rows (first and last included) against the oracle."""
    wl = W.CSA_PREFILL
    qI, w, kI = W.index_queries(wl, DEV), W.index_weights(wl, DEV), W.index_keys(wl, DEV)
    qp = wl.q_positions().to(DEV)
    S = cuda.csa_index(qI, w, kI, qp, wl.m)
    sel = cuda.csa_topk(S, qp, wl.m, wl.k)
    assert cuda.csa_sync_status() == 0
    rows = _prefill_rows(wl.nq)
    rt = torch.from_numpy(rows).to(DEV)
    ref = oracle.index(W.bits(qI[:, rt]), w[:, rt].cpu().numpy(), W.bits(kI), qp[:, rt].cpu().numpy(), wl.m)
    # the kernel's scores on those rows (diagnostic tolerance) and its -inf pattern
    got = f64(S[:, rt])
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    fin = np.isfinite(ref)
    assert np.abs(got[fin] - ref[fin]).max() <= 1e-3 * np.abs(ref[fin]).max()
    check_band(sel[:, rt].cpu().numpy(), ref, qp[:, rt].cpu().numpy(), wl.m, wl.k, wl.N)


# ----------------------------------------------------------------------------- attention at shape
def _causal_selection(q_pos, m, N, k, seed):
    """Seeded selection: k distinct visible entries per query (all when n_vis <= k), -1 padded."""
    r = np.random.default_rng(seed)
    qp = q_pos.reshape(-1)
    idx = np.full((qp.size, k), -1, np.int32)
    for i, t in enumerate(qp):
        nv = oracle.n_visible(int(t), m, N)
        n = min(k, nv)
        idx[i, :n] = np.sort(r.choice(nv, n, replace=False))
    return idx.reshape(q_pos.shape + (k,))


def test_csa_attend_prefill_sampled_rows(cuda):
    """Prefill attention over the whole chunk (4096 queries x 1024 selected
    entries + 128 window rows, 128 heads x 512) in one launch; 24 sampled
    queries against the oracle on the same seeded causal selection."""
    wl = W.CSA_PREFILL
    q = W.queries(wl, DEV)
    kv = W.direct_kv(wl, DEV)
    A = W.stream(wl, "A", 0, DEV).unsqueeze(0)
    qp = wl.q_positions()
    idx = _causal_selection(qp.numpy(), wl.m, wl.N, wl.k, 11)
    out = cuda.csa_attend(q, kv, torch.from_numpy(idx).to(DEV), A, qp.to(DEV), wl.W, wl.scale, wl.eps)
    assert cuda.csa_sync_status() == 0
    rows = _prefill_rows(wl.nq, 24, seed=12)
    rt = torch.from_numpy(rows)
    ref = oracle.attend(W.bits(q[:, rt.to(DEV)]), W.bits(kv), idx[:, rows], W.bits(A), qp[:, rt].numpy(), wl.W,
                        wl.scale, wl.eps)
    got = f64(out[:, rt.to(DEV)])
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


def test_hca_attend_decode_1m_sampled(cuda):
    """HCA decode at its shape: 32 sequences at position 2^20 - 1, 8192 visible
    entries each (m = 128) plus the 128-row window, in one launch; 4 sampled
    sequences (first and last included) against the oracle."""
    wl = W.HCA_DECODE
    q = W.queries(wl, DEV)
    kv = W.direct_kv(wl, DEV)
    win = torch.stack([W.stream(wl, "A", b, DEV, T=wl.W) for b in range(wl.batch)])
    qp = wl.q_positions()
    p0 = wl.T - wl.W
    out = cuda.hca_attend(q, kv, wl.m, win, qp.to(DEV), wl.W, wl.scale, wl.eps, win_pos0=p0)
    assert cuda.csa_sync_status() == 0
    seqs = [0, 11, 22, wl.batch - 1]
    st = torch.tensor(seqs)
    ref = oracle.hca_attend(W.bits(q[st.to(DEV)]), W.bits(kv[st.to(DEV)]), wl.m, W.bits(win[st.to(DEV)]),
                            qp[st].numpy(), wl.W, wl.scale, wl.eps, win_pos0=p0)
    got = f64(out[st.to(DEV)])
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


# ----------------------------------------------------------------------------- FP4 indexer at 1M context
def test_fp4_index_1m_scores_and_recall(cuda):
    """Two sequences of the FP4 workload (262144 entries each, 2 key channels
    x8): FP4 scores against the FP4-exact oracle, the single-pass FP4 top-k in
    the band of the FP4-exact oracle scores, and the recall of the oracle's
    top-k of the bf16-operand scores -- single pass (reported, asserted only
    as >= 0.8: on i.i.d. synthetic data FP4 rounding moves scores across the
    k-th by far more than the band) and after the over-select (4k = 4096) +
    bf16 re-rank path (>= 0.99)."""
    wl = W.FP4_DECODE
    nb = 2
    qI = W.index_queries(wl, DEV)[:nb].contiguous()
    w = W.index_weights(wl, DEV)[:nb].contiguous()
    kI = torch.stack([W.index_keys(wl, DEV, b=b) for b in range(nb)])
    qp = wl.q_positions()[:nb].contiguous().to(DEV)
    q4, q4s = cuda.csa_quantize_fp4(qI)
    k4, k4s = cuda.csa_quantize_fp4(kI)
    S4 = cuda.csa_index_fp4(q4, q4s, w, k4, k4s, qp, wl.m)
    sel1 = cuda.csa_topk(S4, qp, wl.m, wl.k).cpu().numpy()
    cand = cuda.csa_topk(S4, qp, wl.m, 4 * wl.k)
    sel2 = cuda.csa_rescore_topk(qI, w, kI, cand, wl.k).cpu().numpy()
    assert cuda.csa_sync_status() == 0

    qpn, wn = qp.cpu().numpy(), w.cpu().numpy()
    rq4, rq4s = oracle.quantize_fp4(W.bits(qI))
    rk4, rk4s = oracle.quantize_fp4(W.bits(kI))
    assert np.array_equal(rk4, k4.cpu().numpy()) and np.array_equal(rk4s, k4s.cpu().numpy())
    ref4 = oracle.index_fp4(rq4, rq4s, wn, rk4, rk4s, qpn, wl.m)
    got4 = f64(S4)
    assert np.abs(got4 - ref4).max() <= 1e-5 * np.abs(ref4).max()
    check_band(sel1, ref4, qpn, wl.m, wl.k, wl.N)

    ref16 = oracle.index(W.bits(qI), wn, W.bits(kI), qpn, wl.m)
    top16 = oracle.topk(ref16, qpn, wl.m, wl.k)
    r1, r2 = recall(sel1, top16), recall(sel2, top16)
    print("FP4 recall vs the oracle top-%d: single pass %.4f, over-select %d + re-rank %.4f"
          % (wl.k, r1, 4 * wl.k, r2))
    assert r2 >= 0.99, r2
    assert r1 >= 0.8, r1


# ----------------------------------------------------------------------------- the step as one call
@pytest.mark.parametrize("wl", [W.TINY, W.CSA_DECODE], ids=lambda w: w.name)
def test_decode_step_equals_the_three_calls(cuda, wl):
    """csa_decode_step (top-k and attention launched as programmatic dependents)
    gives bit for bit the scores, selection and output of csa_index, csa_topk
    and csa_attend called one after the other, twice in a row."""
    qI, w, kI = W.index_queries(wl, DEV), W.index_weights(wl, DEV), W.index_keys(wl, DEV)
    qp = wl.q_positions().to(DEV)
    q = W.queries(wl, DEV)
    kv = W.direct_kv(wl, DEV)
    win = W.normal_bf16((wl.batch, wl.W, wl.D), 31, DEV)
    p0 = wl.T - wl.W
    S = cuda.csa_index(qI, w, kI, qp, wl.m)
    idx = cuda.csa_topk(S, qp, wl.m, wl.k)
    out = cuda.csa_attend(q, kv, idx, win, qp, wl.W, wl.scale, wl.eps, win_pos0=p0)
    for _ in range(2):
        S2, idx2, out2 = cuda.csa_decode_step(qI, w, kI, q, kv, win, qp, wl.m, wl.k, wl.W, wl.scale, wl.eps,
                                              win_pos0=p0)
        assert cuda.csa_sync_status() == 0
        assert torch.equal(S2, S)
        assert torch.equal(idx2, idx)
        assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
