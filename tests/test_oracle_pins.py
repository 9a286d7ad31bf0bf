"""Pins for the float64 oracle (CPU only).

Each test checks the oracle against something other than itself: a closed
form, an invariant, brute force on a tiny input, an independent library
routine (torch's float8_e4m3fn), or the hyper-parameters printed on the pages.
The tests are chosen so that a plausible slip in the oracle -- a dropped term,
a wrong sign, an off-by-one in the causal threshold, swapped stream halves, a
transposed operand -- fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_06_b200 import workloads as wlmod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x) -> np.ndarray:
    """float array -> bf16 bit patterns (RNE)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_val(bits) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------
# compression
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("m,T", [(4, 37), (3, 12), (1, 5)])
def test_compress_uniform_logits_is_mean_pooling(m, T):
    r = rng(1)
    d = 16
    A = bf16_bits(r.standard_normal((2, T, d)))
    B = bf16_bits(r.standard_normal((2, T, d)))
    L = np.full((2 * m, d), 0.37, np.float32)
    out = oracle.compress(A, B, L, m, apply_rmsnorm=False)
    N = T // m
    assert out.shape == (2, N, d)
    Av, Bv = bf16_val(A), bf16_val(B)
    for b in range(2):
        # entry 0: mean of its m A tokens only (the B half is padded out)
        np.testing.assert_allclose(out[b, 0], Av[b, 0:m].mean(0), rtol=1e-13, atol=1e-14)
        for i in range(1, N):
            rows = np.concatenate([Bv[b, (i - 1) * m:i * m], Av[b, i * m:(i + 1) * m]])
            np.testing.assert_allclose(out[b, i], rows.mean(0), rtol=1e-13, atol=1e-14)


def test_compress_one_hot_logits_select_the_named_row():
    """Channel c puts all its weight on row j=c mod 2m: rows 0..m-1 must be the
    previous m tokens of stream B, rows m..2m-1 the newest m tokens of A."""
    r = rng(2)
    m, T, d = 4, 40, 24
    A = bf16_bits(r.standard_normal((1, T, d)))
    B = bf16_bits(r.standard_normal((1, T, d)))
    L = np.full((2 * m, d), -60.0, np.float32)
    sel = np.arange(d) % (2 * m)
    L[sel, np.arange(d)] = 60.0
    out = oracle.compress(A, B, L, m, apply_rmsnorm=False)[0]
    Av, Bv = bf16_val(A)[0], bf16_val(B)[0]
    for i in range(T // m):
        for c in range(d):
            j = sel[c]
            if i == 0:
                if j < m:   # B half padded: the A logits are all equal -> mean of A rows
                    exp = Av[0:m, c].mean()
                else:
                    exp = Av[j - m, c]
            else:
                exp = Bv[(i - 1) * m + j, c] if j < m else Av[i * m + j - m, c]
            assert abs(out[i, c] - exp) <= 1e-12 * max(1.0, abs(exp)), (i, c)


def test_compress_softmax_shift_invariance_and_linearity():
    r = rng(3)
    m, T, d = 4, 64, 32
    A = r.standard_normal((1, T, d))
    B = r.standard_normal((1, T, d))
    # logits on a 1/64 grid so that adding 3 is exact in fp32
    L = (np.round(r.standard_normal((2 * m, d)) * 64) / 64).astype(np.float32)
    base = oracle.compress(bf16_bits(A), bf16_bits(B), L, m, apply_rmsnorm=False)
    shifted = oracle.compress(bf16_bits(A), bf16_bits(B), L + np.float32(3.0), m, apply_rmsnorm=False)
    np.testing.assert_allclose(shifted, base, rtol=1e-12, atol=1e-13)
    doubled = oracle.compress(bf16_bits(2 * bf16_val(bf16_bits(A))), bf16_bits(2 * bf16_val(bf16_bits(B))),
                              L, m, apply_rmsnorm=False)
    np.testing.assert_allclose(doubled, 2 * base, rtol=1e-13, atol=1e-14)


def test_compress_rmsnorm_closed_form():
    r = rng(4)
    m, T, d = 4, 64, 48
    A = bf16_bits(r.standard_normal((2, T, d)))
    B = bf16_bits(r.standard_normal((2, T, d)))
    L = r.standard_normal((2 * m, d)).astype(np.float32)
    eps = 1e-3
    raw = oracle.compress(A, B, L, m, apply_rmsnorm=False)
    nrm = oracle.compress(A, B, L, m, apply_rmsnorm=True, eps=eps)
    ms = (raw ** 2).mean(-1)
    rms_out = np.sqrt((nrm ** 2).mean(-1))
    np.testing.assert_allclose(rms_out, np.sqrt(ms / (ms + eps)), rtol=1e-12)
    # direction unchanged, gain applied per channel
    np.testing.assert_allclose(nrm * np.sqrt(ms + eps)[..., None], raw, rtol=1e-11, atol=1e-13)
    g = r.uniform(0.5, 2.0, d).astype(np.float32)
    ng = oracle.compress(A, B, L, m, apply_rmsnorm=True, gain=g, eps=eps)
    np.testing.assert_allclose(ng, nrm * g.astype(np.float64), rtol=1e-13)


def test_rmsnorm_rows_closed_form():
    """The row RMSNorm helper: output RMS = sqrt(ms / (ms + eps)) (closed form),
    the direction of every row kept, gain applied per channel, and rows scaled
    by a power of two (exact in bf16) give outputs that follow the closed form
    for their own mean square.  A dropped 1/d, a missing eps, the gain applied
    per row instead of per channel, or a sum of |x| instead of x^2 fails it."""
    r = rng(41)
    rows, d, eps = 37, 48, 1e-2
    x = r.standard_normal((rows, d))
    x[3] *= 2.0 ** -6                      # small rows, where eps matters
    x[5] = 0.0                             # zero row -> zero output, no NaN
    xb = bf16_bits(x)
    xv = bf16_val(xb)
    out = oracle.rmsnorm(xb, eps=eps)
    ms = (xv ** 2).mean(-1)
    np.testing.assert_allclose(np.sqrt((out ** 2).mean(-1)), np.sqrt(ms / (ms + eps)), rtol=1e-12)
    np.testing.assert_allclose(out * np.sqrt(ms + eps)[:, None], xv, rtol=1e-12, atol=1e-300)
    assert np.all(out[5] == 0.0)
    g = r.uniform(0.5, 2.0, d).astype(np.float32)
    np.testing.assert_allclose(oracle.rmsnorm(xb, eps=eps, gain=g), out * g.astype(np.float64), rtol=1e-13)
    # with eps -> 0 the output no longer depends on the row's scale
    big = bf16_bits(xv * 8.0)
    np.testing.assert_allclose(oracle.rmsnorm(big, eps=1e-30), oracle.rmsnorm(xb, eps=1e-30), rtol=1e-12)
    # hand-worked row: x = (3, 4), ms = 12.5, eps = 0 -> x / sqrt(12.5)
    np.testing.assert_allclose(oracle.rmsnorm(bf16_bits([[3.0, 4.0]]), eps=0.0),
                               [[3.0 / math.sqrt(12.5), 4.0 / math.sqrt(12.5)]], rtol=1e-15)


def test_compress_entry_range_matches_full():
    r = rng(5)
    m, T, d = 4, 80, 16
    A = bf16_bits(r.standard_normal((2, T, d)))
    B = bf16_bits(r.standard_normal((2, T, d)))
    L = r.standard_normal((2 * m, d)).astype(np.float32)
    full = oracle.compress(A, B, L, m)
    part = oracle.compress(A, B, L, m, i0=7, ni=5)
    np.testing.assert_array_equal(part, full[:, 7:12])


# input-dependent compression weights Z_a, Z_b ("DeepSeek v4", compressed Key-Value entry)
def test_compress_dynamic_m1_is_a_sigmoid_blend():
    """m = 1: entry i >= 1 pools B[i-1] and A[i] with weight sigma(l_A - l_B) on A,
    l_A = Za[i] + bias[1], l_B = Zb[i-1] + bias[0]; entry 0 is A[0]."""
    r = rng(40)
    T, d = 9, 16
    A, B, Za, Zb = (bf16_bits(r.standard_normal((2, T, d))) for _ in range(4))
    bias = r.standard_normal((2, d)).astype(np.float32)
    out = oracle.compress_dynamic(A, B, Za, Zb, bias, 1, apply_rmsnorm=False)
    Av, Bv, Zav, Zbv = bf16_val(A), bf16_val(B), bf16_val(Za), bf16_val(Zb)
    bb = bias.astype(np.float64)
    np.testing.assert_array_equal(out[:, 0], Av[:, 0])
    for i in range(1, T):
        s = 1.0 / (1.0 + np.exp(-((Zav[:, i] + bb[1]) - (Zbv[:, i - 1] + bb[0]))))
        np.testing.assert_allclose(out[:, i], s * Av[:, i] + (1 - s) * Bv[:, i - 1], rtol=1e-12, atol=1e-14)


def test_compress_dynamic_one_hot_z_selects_the_named_token():
    """Channel c of entry i puts Z = +80 on row j = (i + c) mod 2m and 0 elsewhere:
    the output is that row's token, B[(i-1)m + j] for j < m, A[im + j - m] otherwise
    (entry 0 takes j in the A half)."""
    r = rng(41)
    m, T, d = 4, 42, 24
    A = bf16_bits(r.standard_normal((1, T, d)))
    B = bf16_bits(r.standard_normal((1, T, d)))
    Za = np.zeros((1, T, d), np.float32)
    Zb = np.zeros((1, T, d), np.float32)
    N = T // m
    want = np.empty((N, d))
    Av, Bv = bf16_val(A)[0], bf16_val(B)[0]
    for i in range(N):
        for c in range(d):
            j = (i + c) % (2 * m)
            if i == 0 and j < m:
                j += m
            if j < m:
                Zb[0, (i - 1) * m + j, c] = 80.0
                want[i, c] = Bv[(i - 1) * m + j, c]
            else:
                Za[0, i * m + j - m, c] = 80.0
                want[i, c] = Av[i * m + j - m, c]
    bias = np.zeros((2 * m, d), np.float32)
    out = oracle.compress_dynamic(A, B, bf16_bits(Za), bf16_bits(Zb), bias, m, apply_rmsnorm=False)[0]
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-30)


def test_compress_dynamic_entry0_ignores_the_previous_block():
    """Z_b = +80 on every token: entry 0 (no previous block) is the mean of its A
    rows; every later entry is the mean of its m previous-block B rows."""
    r = rng(42)
    m, T, d = 3, 21, 16
    A = bf16_bits(r.standard_normal((2, T, d)))
    B = bf16_bits(r.standard_normal((2, T, d)))
    Zb = bf16_bits(np.full((2, T, d), 80.0))
    bias = np.zeros((2 * m, d), np.float32)
    out = oracle.compress_dynamic(A, B, None, Zb, bias, m, apply_rmsnorm=False)
    Av, Bv = bf16_val(A), bf16_val(B)
    np.testing.assert_allclose(out[:, 0], Av[:, 0:m].mean(1), rtol=1e-13, atol=1e-15)
    for i in range(1, T // m):
        np.testing.assert_allclose(out[:, i], Bv[:, (i - 1) * m:i * m].mean(1), rtol=1e-12, atol=1e-15)


def test_compress_dynamic_without_z_is_the_static_compress():
    r = rng(43)
    m, T, d = 4, 50, 32
    A = bf16_bits(r.standard_normal((2, T, d)))
    B = bf16_bits(r.standard_normal((2, T, d)))
    bias = r.standard_normal((2 * m, d)).astype(np.float32)
    g = r.uniform(0.5, 2.0, d).astype(np.float32)
    static = oracle.compress(A, B, bias, m, apply_rmsnorm=True, gain=g)
    zeros = np.zeros(A.shape, np.uint16)
    np.testing.assert_allclose(oracle.compress_dynamic(A, B, None, None, bias, m, gain=g), static, rtol=1e-12)
    np.testing.assert_allclose(oracle.compress_dynamic(A, B, zeros, zeros, bias, m, gain=g), static, rtol=1e-12)


def test_compress_dynamic_shift_invariance_and_entry_range():
    """A constant added to every Z value leaves the softmax unchanged; a sub-range
    of entries equals the same rows of the full result."""
    r = rng(44)
    m, T, d = 4, 60, 16
    A = bf16_bits(r.standard_normal((2, T, d)))
    B = bf16_bits(r.standard_normal((2, T, d)))
    # Z on a 1/8 grid in [-3, 3]: +2 stays exact in bf16
    Za = np.clip(np.round(r.standard_normal((2, T, d)) * 8) / 8, -3, 3)
    Zb = np.clip(np.round(r.standard_normal((2, T, d)) * 8) / 8, -3, 3)
    bias = r.standard_normal((2 * m, d)).astype(np.float32)
    base = oracle.compress_dynamic(A, B, bf16_bits(Za), bf16_bits(Zb), bias, m)
    shifted = oracle.compress_dynamic(A, B, bf16_bits(Za + 2), bf16_bits(Zb + 2), bias, m)
    np.testing.assert_allclose(shifted, base, rtol=1e-12, atol=1e-14)
    part = oracle.compress_dynamic(A, B, bf16_bits(Za), bf16_bits(Zb), bias, m, i0=6, ni=5)
    np.testing.assert_array_equal(part, base[:, 6:11])


# ----------------------------------------------------------------------------
# indexer
# ----------------------------------------------------------------------------
def test_index_parallel_keys_closed_form():
    """q_h = c_h * k with integer c_h: score = sum_{c_h > 0} w_h c_h |k|^2 (ReLU drops c_h < 0)."""
    r = rng(6)
    H_I, d_I, N, m = 5, 16, 12, 4
    k = r.integers(-2, 3, size=(1, N, d_I)).astype(np.float64)
    c = np.array([2.0, -1.0, 3.0, -4.0, 1.0])
    s_ref = 7  # queries parallel to key 7
    q = c[:, None] * k[0, s_ref][None, :]
    w = np.array([[[0.5, 2.0, 0.25, 1.0, 1.5]]], np.float32)
    T = N * m
    S = oracle.index(bf16_bits(q[None, None]), w, bf16_bits(k), np.array([[T - 1]], np.int32), m)
    expect = float(np.sum(np.where(c > 0, w[0, 0] * c, 0.0))) * float(k[0, s_ref] @ k[0, s_ref])
    assert S[0, 0, s_ref] == pytest.approx(expect, rel=1e-15)
    # a key orthogonal to every query head scores exactly 0
    k2 = np.zeros((1, N, d_I))
    k2[0, :, 0] = 1.0
    q2 = np.zeros((H_I, d_I))
    q2[:, 1] = r.standard_normal(H_I)
    S2 = oracle.index(bf16_bits(q2[None, None]), w, bf16_bits(k2), np.array([[T - 1]], np.int32), m)
    assert np.all(S2 == 0.0)
    # all dot products negative -> 0
    S3 = oracle.index(bf16_bits(-np.abs(q2)[None, None] - 1), w, bf16_bits(np.abs(k2)),
                      np.array([[T - 1]], np.int32), m)
    assert np.all(S3 == 0.0)


def test_index_weights_are_linear_per_head():
    r = rng(7)
    H_I, d_I, N, m = 3, 8, 10, 2
    q = bf16_bits(r.standard_normal((1, 1, H_I, d_I)))
    k = bf16_bits(r.standard_normal((1, N, d_I)))
    pos = np.array([[N * m - 1]], np.int32)
    per_head = []
    for h in range(H_I):
        e = np.zeros((1, 1, H_I), np.float32)
        e[0, 0, h] = 1.0
        per_head.append(oracle.index(q, e, k, pos, m))
    w = np.array([[[0.5, 0.25, 2.0]]], np.float32)
    S = oracle.index(q, w, k, pos, m)
    np.testing.assert_allclose(S, sum(w[0, 0, h] * per_head[h] for h in range(H_I)), rtol=1e-14)
    assert all(np.all(p >= 0) for p in per_head)


@pytest.mark.parametrize("m", [1, 4, 128])
def test_index_causal_threshold(m):
    r = rng(8)
    N = 9
    T = N * m
    q = bf16_bits(r.standard_normal((1, 4, 2, 8)))
    w = np.ones((1, 4, 2), np.float32)
    k = bf16_bits(r.standard_normal((1, N, 8)))
    # positions: before the first entry completes, exactly at an entry boundary, last token
    ts = [m - 2 if m >= 2 else 0, m - 1, 3 * m - 1, T - 1]
    pos = np.array([ts], np.int32)
    S = oracle.index(q, w, k, pos, m)
    for i, t in enumerate(ts):
        nv = (t + 1) // m
        assert np.all(np.isfinite(S[0, i, :nv]))
        assert np.all(np.isneginf(S[0, i, nv:]))


# ----------------------------------------------------------------------------
# top-k
# ----------------------------------------------------------------------------
def _better(scores, a, b):
    return scores[a] > scores[b] or (scores[a] == scores[b] and a < b)


@pytest.mark.parametrize("seed", range(5))
def test_topk_matches_rank_counting_brute_force(seed):
    r = rng(100 + seed)
    N, m, k = 23, 1, 6
    scores = r.integers(0, 5, size=(1, 3, N)).astype(np.float64)   # many ties
    scores[0, 1] = r.standard_normal(N)
    pos = np.array([[N - 1, 10, 4]], np.int32)
    idx = oracle.topk(scores, pos, m, k)
    for q in range(3):
        nv = (pos[0, q] + 1) // m
        s = scores[0, q]
        chosen = {int(v) for v in idx[0, q] if v >= 0}
        # s is chosen iff fewer than k visible entries rank strictly better
        brute = {a for a in range(nv) if sum(_better(s, b, a) for b in range(nv)) < k}
        assert chosen == brute
        assert sum(v == -1 for v in idx[0, q]) == max(0, k - nv)
        assert list(idx[0, q][: min(k, nv)]) == sorted(chosen, key=lambda a: (-s[a], a))


def test_topk_permutation_equivariance():
    r = rng(9)
    N, k = 50, 7
    s = r.standard_normal(N)
    perm = r.permutation(N)
    pos = np.array([[N - 1]], np.int32)
    a = oracle.topk(s[None, None], pos, 1, k)[0, 0]
    b = oracle.topk(s[perm][None, None], pos, 1, k)[0, 0]
    assert {int(perm[i]) for i in b} == {int(i) for i in a}


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def _attn_inputs(r, batch=1, nq=1, H=4, D=32, N=20, T=40):
    q = bf16_bits(r.standard_normal((batch, nq, H, D)))
    kv = bf16_bits(r.standard_normal((batch, N, D)))
    win = bf16_bits(r.standard_normal((batch, T, D)))
    return q, kv, win


def test_attend_single_key_returns_it():
    r = rng(10)
    q, kv, win = _attn_inputs(r)
    idx = np.full((1, 1, 5), -1, np.int32)
    t = 17
    out = oracle.attend(q, kv, idx, win, np.array([[t]], np.int32), W=1, scale=0.3)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(bf16_val(win)[0, t], out[0, 0].shape), rtol=1e-15)


def test_attend_identical_keys_return_the_key():
    r = rng(11)
    H, D, N, T = 4, 32, 20, 40
    q = bf16_bits(r.standard_normal((1, 1, H, D)))
    x = r.standard_normal(D)
    kv = bf16_bits(np.broadcast_to(x, (1, N, D)))
    win = bf16_bits(np.broadcast_to(x, (1, T, D)))
    idx = np.array([[[3, 9, -1, 14, 0]]], np.int32)
    out = oracle.attend(q, kv, idx, win, np.array([[30]], np.int32), W=8, scale=1.0)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(bf16_val(kv)[0, 0], (H, D)), rtol=1e-14)


def test_attend_zero_scale_is_mean_of_key_set_and_window_clips_at_zero():
    r = rng(12)
    q, kv, win = _attn_inputs(r)
    idx = np.array([[[2, -1, 11, 5, 99]]], np.int32)    # -1 and out-of-range ignored
    t, W = 3, 16                                          # window clipped to rows 0..3
    out = oracle.attend(q, kv, idx, win, np.array([[t]], np.int32), W=W, scale=0.0)
    rows = np.concatenate([bf16_val(kv)[0, [2, 11, 5]], bf16_val(win)[0, 0:t + 1]])
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(rows.mean(0), out[0, 0].shape), rtol=1e-13, atol=1e-15)


def test_attend_equal_logits_cancel():
    """q orthogonal to both keys (+x and -x): equal logits, output 0."""
    H, D = 2, 16
    q = np.zeros((1, 1, H, D))
    q[..., 0] = 1.0
    x = np.linspace(-1, 1, D)
    x[0] = 0.0
    kv = bf16_bits(np.stack([x, -x])[None])
    win = bf16_bits(np.zeros((1, 4, D)))
    idx = np.array([[[0, 1]]], np.int32)
    # window rows are zero vectors: q.x = 0 too, so every logit is 0 and the
    # output is (x - x + 0)/3 = 0
    out = oracle.attend(bf16_bits(q), kv, idx, win, np.array([[1]], np.int32), W=1, scale=5.0)
    assert np.max(np.abs(out)) < 1e-15


def test_attend_large_scale_picks_the_best_key():
    r = rng(13)
    H, D, N = 3, 16, 6
    kvf = r.standard_normal((1, N, D))
    kvb = bf16_bits(kvf)
    kvv = bf16_val(kvb)
    q = np.broadcast_to(kvv[0, 4], (1, 1, H, D))       # q parallel to entry 4
    win = bf16_bits(np.zeros((1, 2, D)))
    idx = np.arange(N, dtype=np.int32)[None, None]
    out = oracle.attend(bf16_bits(q), kvb, idx, win, np.array([[0]], np.int32), W=1, scale=1e4)
    best = int(np.argmax(kvv[0] @ kvv[0, 4]))
    assert best == 4
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(kvv[0, 4], (H, D)), rtol=1e-12, atol=1e-12)


def test_attend_query_rmsnorm_makes_query_scale_irrelevant():
    r = rng(14)
    q, kv, win = _attn_inputs(r, H=3, D=32)
    idx = np.array([[[1, 4, 7, -1]]], np.int32)
    pos = np.array([[25]], np.int32)
    a = oracle.attend(q, kv, idx, win, pos, W=6, scale=0.2, eps=0.0)
    q4 = bf16_bits(4.0 * bf16_val(q))
    b = oracle.attend(q4, kv, idx, win, pos, W=6, scale=0.2, eps=0.0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_attend_sink_single_key_is_a_sigmoid():
    """One all-ones key and an all-ones query: the key's logit is
    a = scale * D / sqrt(1 + eps), and with a sink logit c the key keeps the
    weight e^a / (e^a + e^c) = sigmoid(a - c) -- a closed form."""
    H, D, eps = 3, 16, 1e-6
    q = bf16_bits(np.ones((1, 1, H, D)))
    win = bf16_bits(np.ones((1, 8, D)))
    idx = np.full((1, 1, 2), -1, np.int32)
    scale = 1.0 / D
    a = scale * D / math.sqrt(1.0 + eps)
    sinks = np.array([-2.0, 0.5, 3.0], np.float32)
    out = oracle.attend(q, win, idx, win, np.array([[5]], np.int32), W=1, scale=scale, eps=eps, sinks=sinks)
    for h in range(H):
        want = 1.0 / (1.0 + math.exp(float(sinks[h]) - a))
        np.testing.assert_allclose(out[0, 0, h], np.full(D, want), rtol=1e-12)


def test_attend_sink_at_minus_infinity_is_no_sink_and_a_huge_sink_silences():
    r = rng(16)
    q, kv, win = _attn_inputs(r)
    idx = np.array([[[2, 7, -1, 11]]], np.int32)
    pos = np.array([[33]], np.int32)
    base = oracle.attend(q, kv, idx, win, pos, W=6, scale=0.2)
    none = oracle.attend(q, kv, idx, win, pos, W=6, scale=0.2, sinks=np.full(4, -np.inf, np.float32))
    assert np.array_equal(base, none)
    loud = oracle.attend(q, kv, idx, win, pos, W=6, scale=0.2, sinks=np.full(4, 1e4, np.float32))
    assert np.abs(loud).max() == 0.0


# partial RoPE ("DeepSeek-V4-Pro - Model techniques map", "Partial RoPE" and the
# rope-conjugate rotation of the attention output)
def _rope_tables(n_pos, r, seed=0, omega=None):
    """cos / sin of angles p * omega_i for p < n_pos (omega drawn if not given)."""
    om = rng(seed).uniform(0.01, 1.5, r) if omega is None else np.asarray(omega, np.float64)
    ang = np.arange(n_pos)[:, None] * om[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def test_rope_hand_worked_example():
    """width 6 = 2 unrotated + 4 rotated channels, r = 2; at position 1 the
    angles are (pi/2, 0): rotate_half pairs channel 2 with 4 and 3 with 5, so
    x = [5, 6, 1, 2, 3, 4] -> [5, 6, 1*0 - 3*1, 2, 3*0 + 1*1, 4] = [5, 6, -3, 2, 1, 4]
    and the conjugate gives [5, 6, 3, 2, -1, 4]; position 0 (angle 0) is the identity."""
    cos = np.array([[1, 1], [0, 1]], np.float32)
    sin = np.array([[0, 0], [1, 0]], np.float32)
    x = np.array([5, 6, 1, 2, 3, 4], np.float64)
    np.testing.assert_array_equal(oracle.rope(x, 1, cos, sin), [5, 6, -3, 2, 1, 4])
    np.testing.assert_array_equal(oracle.rope(x, 1, cos, sin, inverse=True), [5, 6, 3, 2, -1, 4])
    np.testing.assert_array_equal(oracle.rope(x, 0, cos, sin), x)


def test_rope_is_complex_multiplication_of_half_pairs():
    """Independent route: the rotated slice equals (x1 + i x2) * exp(i theta)
    computed with numpy complex arithmetic; the unrotated channels are kept."""
    r_, width = 32, 96
    cos, sin = _rope_tables(50, r_, seed=1)
    x = rng(2).standard_normal((7, width))
    pos = np.array([0, 1, 7, 13, 31, 48, 49], np.int32)
    y = oracle.rope(x, pos, cos, sin)
    n = width - 2 * r_
    z = (x[:, n:n + r_] + 1j * x[:, n + r_:]) * (cos[pos].astype(np.float64) + 1j * sin[pos].astype(np.float64))
    np.testing.assert_array_equal(y[:, :n], x[:, :n])
    np.testing.assert_allclose(y[:, n:n + r_], z.real, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(y[:, n + r_:], z.imag, rtol=1e-13, atol=1e-14)


def test_rope_preserves_norm_inverse_undoes_and_scores_see_relative_position():
    r_, width = 16, 64
    cos, sin = _rope_tables(64, r_, seed=3)
    g = rng(4)
    q, k = g.standard_normal(width), g.standard_normal(width)
    y = oracle.rope(q, 9, cos, sin)
    # fp32 tables: cos^2 + sin^2 = 1 to ~1e-7, so norm and inverse hold to that
    assert abs(np.linalg.norm(y) - np.linalg.norm(q)) < 2e-7 * np.linalg.norm(q)
    np.testing.assert_allclose(oracle.rope(y, 9, cos, sin, inverse=True), q, rtol=0, atol=4e-7 * np.abs(q).max())
    # (R_t q) . (R_s k) depends on t - s only (angles p * omega); fp32 tables limit the agreement
    d1 = oracle.rope(q, 20, cos, sin) @ oracle.rope(k, 5, cos, sin)
    d2 = oracle.rope(q, 40, cos, sin) @ oracle.rope(k, 25, cos, sin)
    assert abs(d1 - d2) < 1e-5 * (np.linalg.norm(q) * np.linalg.norm(k))


def test_attend_rope_identity_tables_equal_no_rope():
    r = rng(17)
    q, kv, win = _attn_inputs(r, H=4, D=32)
    idx = np.array([[[2, 7, -1, 11]]], np.int32)
    pos = np.array([[33]], np.int32)
    cos = np.ones((40, 8), np.float32)
    sin = np.zeros((40, 8), np.float32)
    base = oracle.attend(q, kv, idx, win, pos, W=6, scale=0.2)
    np.testing.assert_array_equal(oracle.attend(q, kv, idx, win, pos, W=6, scale=0.2, rope=(cos, sin)), base)


def test_attend_rope_single_key_is_its_conjugate_rotation():
    """One key (the window row at t): weight 1, so the output is that row
    rotated back by the conjugate at the query position."""
    r = rng(18)
    q, kv, win = _attn_inputs(r, H=3, D=32)
    cos, sin = _rope_tables(40, 8, seed=5)
    t = 17
    idx = np.full((1, 1, 3), -1, np.int32)
    out = oracle.attend(q, kv, idx, win, np.array([[t]], np.int32), W=1, scale=0.3, rope=(cos, sin))
    x = bf16_val(win)[0, t]
    n = 32 - 16
    z = (x[n:n + 8] + 1j * x[n + 8:]) * (cos[t].astype(np.float64) - 1j * sin[t].astype(np.float64))
    want = np.concatenate([x[:n], z.real, z.imag])
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(want, (3, 32)), rtol=1e-13, atol=1e-14)


def test_attend_rope_output_sees_relative_positions_only():
    """Angles that are multiples of pi/2 keep every rotation exact in bf16.
    Keys rotated at their positions s_j and the query at t give the same output
    as everything shifted by one position: logits and the conjugated values
    depend on s_j - t only.  A missing or misplaced conjugate breaks this."""
    H, D, r_ = 2, 16, 4
    cos, sin = _rope_tables(64, r_, omega=[np.pi / 2, np.pi, 3 * np.pi / 2, np.pi / 2])
    cos, sin = np.round(cos), np.round(sin)
    g = rng(19)
    q = bf16_bits(g.standard_normal((1, 1, H, D)))
    raw = bf16_val(bf16_bits(g.standard_normal((30, D))))
    s_pos = np.arange(30)

    def run(shift):
        rows = oracle.rope(raw, s_pos + shift, cos, sin)       # exact: entries are permuted / negated
        win = bf16_bits(rows)[None]
        t = 25 + shift
        idx = np.full((1, 1, 2), -1, np.int32)
        return oracle.attend(q, win, idx, win, np.array([[t]], np.int32), W=8, scale=0.5, win_pos0=shift,
                             rope=(cos, sin))

    a, b = run(0), run(1)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    assert np.abs(a[..., D - 2 * r_:]).max() > 0.1   # the rotated channels carry signal


def test_hca_equals_csa_with_every_visible_entry():
    r = rng(15)
    m, N, T, W = 4, 12, 48, 5
    q, kv, win = _attn_inputs(r, nq=3, N=N, T=T)
    pos = np.array([[47, 20, 2]], np.int32)
    hca = oracle.hca_attend(q, kv, m, win, pos, W, scale=0.25)
    k = N + 3
    idx = np.full((1, 3, k), -1, np.int32)
    for i, t in enumerate(pos[0]):
        nv = (t + 1) // m
        idx[0, i, :nv] = np.arange(nv)
    csa = oracle.attend(q, kv, idx, win, pos, W, scale=0.25)
    np.testing.assert_allclose(hca, csa, rtol=1e-13, atol=1e-15)
    # the selection order does not matter
    idx2 = idx.copy()
    idx2[0, 0, :N] = idx2[0, 0, :N][::-1]
    np.testing.assert_allclose(oracle.attend(q, kv, idx2, win, pos, W, scale=0.25), csa,
                               rtol=1e-13, atol=1e-15)
    # and with partial RoPE on both sides
    rope = _rope_tables(T, 8, seed=6)
    np.testing.assert_allclose(oracle.hca_attend(q, kv, m, win, pos, W, scale=0.25, rope=rope),
                               oracle.attend(q, kv, idx, win, pos, W, scale=0.25, rope=rope), rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------------------
# FP4 (e2m1 elements, e4m3 block scales)
# ----------------------------------------------------------------------------
def test_e2m1_decode_from_bit_fields():
    for code in range(16):
        sign = -1.0 if code & 8 else 1.0
        e, mt = (code >> 1) & 3, code & 1
        val = mt * 0.5 if e == 0 else (1 + mt / 2) * 2.0 ** (e - 1)
        assert oracle.e2m1_decode(code) == sign * val


def test_e4m3_decode_matches_torch_float8_e4m3fn_exhaustively():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(1) == 2.0 ** -9


def test_e4m3_encode_matches_torch_rounding():
    r = rng(16)
    x = np.concatenate([
        np.exp(r.uniform(np.log(2.0 ** -12), np.log(440.0), 4000)),
        # exact midpoints between neighbouring codes (ties -> even mantissa)
        [(oracle.e4m3_decode(c) + oracle.e4m3_decode(c + 1)) / 2 for c in range(0, 0x7D)],
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    assert np.array_equal(ref, got)
    assert oracle.e4m3_encode(1000.0) == 0x7E      # satfinite
    assert oracle.e4m3_encode(0.0) == 0


def _e2m1_rne_reference(x: float) -> float:
    """Round-half-even on the e2m1 grid written as three uniform sub-grids."""
    a = min(abs(x), 6.0)
    step = 0.5 if a < 2 else (1.0 if a < 4 else 2.0)
    qv = a / step
    fl = math.floor(qv)
    frac = qv - fl
    n = fl + (1 if frac > 0.5 or (frac == 0.5 and fl % 2 == 1) else 0)
    return n * step


def test_e2m1_encode_round_half_even():
    r = rng(17)
    xs = list(r.uniform(-7, 7, 3000)) + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.25, -5.0, -0.1]
    for x in xs:
        x32 = float(np.float32(x))
        code = oracle.e2m1_encode(x32)
        mag = _e2m1_rne_reference(x32)
        assert abs(oracle.e2m1_decode(code)) == mag, x32
        assert (code & 8) == (8 if (x32 < 0 and mag != 0) else 0)
    assert oracle.e2m1_encode(0.25) == 0 and oracle.e2m1_encode(0.75) == 2
    assert oracle.e2m1_encode(2.5) == 4 and oracle.e2m1_encode(5.0) == 6
    assert oracle.e2m1_encode(-0.1) == 0          # a zero magnitude is stored as +0


def test_fp4_round_trip_of_representable_blocks():
    r = rng(18)
    rows, d = 6, 64
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    vals = np.zeros((rows, d))
    scales = []
    for row in range(rows):
        for blk in range(d // 16):
            sc = int(r.integers(0x20, 0x50))            # a normal e4m3 scale
            s = oracle.e4m3_decode(sc)
            codes = r.integers(0, 8, 16)
            codes[r.integers(0, 16)] = 7                  # block max is 6 * s
            sign = np.where(r.random(16) < 0.5, -1.0, 1.0)
            vals[row, blk * 16:(blk + 1) * 16] = sign * grid[codes] * s
            scales.append(sc)
    xb = bf16_bits(vals)
    assert np.array_equal(bf16_val(xb), vals)             # exactly representable in bf16
    packed, sc = oracle.quantize_fp4(xb)
    assert list(sc.reshape(-1)) == scales
    np.testing.assert_array_equal(oracle.dequantize_fp4(packed, sc), vals)


def test_fp4_zero_block_and_packing_order():
    x = np.zeros((1, 32))
    x[0, 16] = 6.0     # second block: element 0 -> low nibble of byte 8
    x[0, 17] = -3.0    # element 1 -> high nibble
    packed, sc = oracle.quantize_fp4(bf16_bits(x))
    assert sc[0, 0] == 0 and np.all(packed[0, :8] == 0)
    assert oracle.e4m3_decode(int(sc[0, 1])) == 1.0
    assert packed[0, 8] == (0x7 | (0xD << 4))


# FP8 KV cache ("DeepSeek-V4-Pro - Model techniques map", inference quantization)
def _fp8_rows(seed, rows=6, d=256):
    r = rng(seed)
    x = r.standard_normal((rows, d)) * np.exp(r.uniform(-6, 6, (rows, 1)))   # rows of very different sizes
    x[1, 128:] = 0.0                                                          # an all-zero block
    x[2, :128] = 0.0
    x[2, 5] = 2.0 ** -20                                                      # a tiny block
    return bf16_bits(x)


def test_fp8_kv_codes_match_torch_float8_with_the_tightest_power_of_two_scale():
    """Independent route: the scale from frexp (smallest 2^k >= absmax/448) and
    the codes from torch's float8_e4m3fn cast of x / 2^k (round-half-even)."""
    x = _fp8_rows(30)
    codes, exps = oracle.quantize_fp8_kv(x, 128)
    xv = bf16_val(x)
    for r_ in range(x.shape[0]):
        for blk in range(2):
            seg = xv[r_, blk * 128:(blk + 1) * 128]
            amax = np.abs(seg).max()
            if amax == 0.0:
                assert exps[r_, blk] == 127 and not codes[r_, blk * 128:(blk + 1) * 128].any()
                continue
            mant, ex = np.frexp(amax / 448.0)        # amax/448 = mant * 2^ex, mant in [0.5, 1)
            k = ex - 1 if mant == 0.5 else ex
            assert exps[r_, blk] == k + 127
            assert 224.0 < amax / 2.0 ** k <= 448.0
            ref = torch.from_numpy((seg / 2.0 ** k).astype(np.float32)).to(torch.float8_e4m3fn)
            got = codes[r_, blk * 128:(blk + 1) * 128]
            refv = ref.to(torch.float64).numpy()
            gotv = np.array([oracle.e4m3_decode(c) for c in got])
            assert np.array_equal(refv, gotv), (r_, blk)


def test_fp8_kv_dequantised_values_are_bf16_and_within_half_an_e4m3_step():
    x = _fp8_rows(31)
    codes, exps = oracle.quantize_fp8_kv(x, 128)
    dq = oracle.dequantize_fp8_kv(codes, exps, 128)
    np.testing.assert_array_equal(bf16_val(bf16_bits(dq)), dq)            # exactly representable in bf16
    xv = bf16_val(x)
    s = np.repeat(2.0 ** (exps.astype(np.float64) - 127), 128, axis=-1)
    bound = np.maximum(2.0 ** -4 * np.abs(xv), 2.0 ** -10 * s)              # half a step, normal / subnormal
    assert np.all(np.abs(dq - xv) <= bound)


def test_fp8_kv_extreme_blocks_keep_every_value_a_finite_bf16():
    """A block of bf16's smallest subnormals and one near its largest value:
    the scale exponent is clamped to [-124, 119], so the dequantised values
    stay exact bf16 numbers and finite."""
    tiny = np.full((1, 128), 2.0 ** -133)
    tiny[0, 1::2] = 3 * 2.0 ** -133
    big = np.full((1, 128), 1.9921875 * 2.0 ** 127)    # bf16's largest value: it would need k = 120
    x = bf16_bits(np.concatenate([tiny, big], axis=1))
    codes, exps = oracle.quantize_fp8_kv(x, 128)
    assert list(exps[0]) == [127 - 124, 127 + 119]
    dq = oracle.dequantize_fp8_kv(codes, exps, 128)
    assert np.all(np.isfinite(dq))
    np.testing.assert_array_equal(bf16_val(bf16_bits(dq)), dq)
    np.testing.assert_array_equal(dq[0, :128], bf16_val(x)[0, :128])   # 2^-133 = code 2^-9 at s = 2^-124
    assert np.all(dq[0, 128:] == 448.0 * 2.0 ** 119)                    # saturated


def test_fp8_kv_round_trip_of_representable_rows():
    """Rows built from e4m3 values times a power of two whose block maximum is
    448 * 2^k come back exactly."""
    r = rng(32)
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])
    rows = []
    for k in (-9, 0, 5):
        v = r.choice(vals, 256) * r.choice([-1.0, 1.0], 256)
        v[0] = 448.0
        v[128] = -448.0
        rows.append(v * 2.0 ** k)
    x = bf16_bits(np.array(rows))
    codes, exps = oracle.quantize_fp8_kv(x, 128)
    np.testing.assert_array_equal(oracle.dequantize_fp8_kv(codes, exps, 128), bf16_val(x))
    assert list(exps[:, 0]) == [127 - 9, 127, 127 + 5]


def test_fp4_index_equals_bf16_index_on_dequantised_operands():
    r = rng(19)
    b, nq, H_I, d_I, N, m = 2, 2, 4, 32, 16, 4
    qx = bf16_bits(r.standard_normal((b, nq, H_I, d_I)))
    kx = bf16_bits(r.standard_normal((b, N, d_I)) * np.where(np.arange(d_I) == 5, 8.0, 1.0))
    q4, q4s = oracle.quantize_fp4(qx)
    k4, k4s = oracle.quantize_fp4(kx)
    w = r.random((b, nq, H_I)).astype(np.float32)
    pos = np.array([[N * m - 1, 30]] * b, np.int32)
    s4 = oracle.index_fp4(q4, q4s, w, k4, k4s, pos, m)
    qd, kd = oracle.dequantize_fp4(q4, q4s), oracle.dequantize_fp4(k4, k4s)
    assert np.array_equal(bf16_val(bf16_bits(qd)), qd) and np.array_equal(bf16_val(bf16_bits(kd)), kd)
    s16 = oracle.index(bf16_bits(qd), w, bf16_bits(kd), pos, m)
    np.testing.assert_allclose(s4, s16, rtol=1e-15)
    assert np.isneginf(s4[0, 1, (30 + 1) // m:]).all()


# ----------------------------------------------------------------------------
# workloads use the printed hyper-parameters
# ----------------------------------------------------------------------------
def test_workloads_use_the_pages_hyperparameters():
    g = json.load(open(os.path.join(GOLDEN, "v4_hyperparams.json")))
    for wl in (wlmod.CSA_DECODE, wlmod.CSA_PREFILL, wlmod.FP4_DECODE):
        assert wl.k == g["index_topk"]["value"]
        assert (wl.H_I, wl.d_I) == (g["index_n_heads"]["value"], g["index_head_dim"]["value"])
        assert wl.m == 4 and wl.m in g["compress_ratios"]["value"]
    for wl in (wlmod.CSA_DECODE, wlmod.CSA_PREFILL, wlmod.HCA_DECODE, wlmod.FP4_DECODE):
        assert wl.W == g["sliding_window"]["value"]
        assert (wl.H, wl.D) == (g["num_attention_heads"]["value"], g["head_dim"]["value"])
    assert wlmod.HCA_DECODE.m == 128 and 128 in g["compress_ratios"]["value"]
    assert wlmod.CSA_DECODE.N == 32768 and wlmod.HCA_DECODE.N == 8192 and wlmod.FP4_DECODE.N == 262144


def test_tiny_workload_end_to_end_consistency():
    """The oracle's chain on the tiny workload: k >= visible collapses CSA to HCA,
    and the top-k entries have the largest scores."""
    wl = wlmod.TINY
    A, B = wlmod.streams(wl)
    L = wlmod.pool_logits(wl)
    C = oracle.compress(wlmod.bits(A), wlmod.bits(B), L.numpy(), wl.m)
    assert C.shape == (1, wl.N, wl.D)
    np.testing.assert_allclose(np.sqrt((C ** 2).mean(-1)), 1.0, rtol=1e-5)
    qI, w, kI = wlmod.index_queries(wl), wlmod.index_weights(wl), wlmod.index_keys(wl)
    pos = wl.q_positions().numpy()
    S = oracle.index(wlmod.bits(qI), w.numpy(), wlmod.bits(kI), pos, wl.m)
    idx = oracle.topk(S, pos, wl.m, wl.k)
    sel = idx[0, 0]
    assert np.all(sel >= 0) and len(set(sel.tolist())) == wl.k
    assert S[0, 0, sel].min() >= np.sort(S[0, 0])[::-1][wl.k - 1]
