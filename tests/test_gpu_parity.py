"""GPU parity: every kernel, called through the C ABI, against the float64
oracle on the same seeded input bits.

Tolerances (the arithmetic is fp32 on bf16/FP4 inputs; a bf16 output carries
a relative rounding error of at most 2^-9):
  * compress: |gpu - oracle| <= 8e-3 * max|oracle row| per entry;
  * index (bf16): |gpu - oracle| <= 1e-3 * max|S| per query (fp32 sums of 128
    products, 64 heads), -inf pattern exact;
  * top-k on identical fp32 scores: identical index sets (both sides break
    ties towards the lower index), ascending order, same number of -1 slots;
  * top-k on the kernel's own scores vs the oracle's float64 scores: the set
    difference may only hold entries within 1e-4 * |s_k| of the k-th score;
  * attention: max|err| <= 2e-2 * max|out| against the oracle on the same
    selection;
  * FP4 quantisation: bit-exact codes and scales; FP4 scores: 1e-5 * max|S|
    (products are exact, only the fp32 summation order differs).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_06_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


def bits(t):
    return W.bits(t)


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def seeded(shape, seed, kind="normal"):
    if kind == "normal":
        return W.normal_bf16(shape, seed, DEV)
    return W.uniform_f32(shape, seed, DEV)


def positions(batch, nq, ts):
    return torch.tensor(np.array(ts, np.int32).reshape(batch, nq), device=DEV)


# ----------------------------------------------------------------------------- compress
@pytest.mark.parametrize("batch,T,d,m,rms,use_gain", [
    (1, 2048, 64, 4, True, False),      # tiny workload shape
    (2, 1037, 512, 4, True, True),      # ragged T, V4 width
    (2, 777, 64, 3, False, False),      # odd m, no norm
    (1, 4 * 128 + 77, 512, 128, True, False),   # HCA ratio (chunked large-m kernel), ragged tail
    (2, 300, 256, 16, True, True),
    (3, 5, 64, 4, True, False),         # N = 1
    (1, 1000, 1024, 64, True, False),   # chunked large-m kernel, 8-row chunks
    (1, 1000, 256, 20, True, True),     # chunked large-m kernel, a partial last chunk
    (1, 3 * 160 + 50, 128, 160, True, False),   # online-softmax kernel (d = 128)
    (2, 128 * 37 + 5, 512, 128, True, True),    # chunked large-m kernel: two sequences, a partial entry group
    (3, 40 * 9 + 3, 1024, 40, True, False),     # chunked large-m kernel, three sequences, 8-row chunks
])
def test_compress_parity(cuda, batch, T, d, m, rms, use_gain):
    A = seeded((batch, T, d), 11)
    B = seeded((batch, T, d), 12)
    L = torch.randn((2 * m, d), generator=torch.Generator(DEV).manual_seed(13), device=DEV)
    gain = (seeded((d,), 14, "uniform") + 0.5) if use_gain else None
    out = cuda.csa_compress(A, B, L, m, rms, gain, 1e-6)
    ref = oracle.compress(bits(A), bits(B), L.cpu().numpy(), m, rms,
                          None if gain is None else gain.cpu().numpy(), 1e-6)
    got = f64(out)
    assert got.shape == ref.shape
    err = np.abs(got - ref).max(-1)
    assert np.all(err <= 8e-3 * np.abs(ref).max(-1)), err.max()


def test_compress_m1_one_hot_logits_is_row_rmsnorm(cuda):
    """m = 1 with logits (-inf for the B row, 0 for the A row) pools each A row
    alone: the result is the row RMSNorm of A (how the FP4 workload normalises
    its directly drawn compressed rows), against the oracle's RMSNorm."""
    A = seeded((2, 333, 512), 15)
    B = seeded((2, 333, 512), 16)
    one = torch.cat([torch.full((1, 512), float("-inf"), device=DEV), torch.zeros((1, 512), device=DEV)])
    out = cuda.csa_compress(A, B, one, 1)
    ref = oracle.rmsnorm(bits(A), eps=1e-6)
    _check_rows(f64(out), ref)


# ----------------------------------------------------------------------------- compress, input-dependent weights
def _dyn_inputs(batch, T, d, m, z_scale=1.0, seed=60):
    A = seeded((batch, T, d), seed)
    B = seeded((batch, T, d), seed + 1)
    Za = (seeded((batch, T, d), seed + 2).float() * z_scale).to(torch.bfloat16)
    Zb = (seeded((batch, T, d), seed + 3).float() * z_scale).to(torch.bfloat16)
    bias = torch.randn((2 * m, d), generator=torch.Generator(DEV).manual_seed(seed + 4), device=DEV)
    return A, B, Za, Zb, bias


def _check_rows(got, ref):
    assert got.shape == ref.shape
    err = np.abs(got - ref).max(-1)
    assert np.all(err <= 8e-3 * np.abs(ref).max(-1)), err.max()


@pytest.mark.parametrize("batch,T,d,m,rms,use_gain,za,zb,z_scale", [
    (1, 2048, 64, 4, True, False, True, True, 1.0),       # tiny workload shape
    (2, 1037, 512, 4, True, True, True, True, 1.0),       # V4 width (warp reduction), ragged T
    (2, 777, 64, 3, False, False, True, False, 1.0),      # odd m, no norm, Zb absent
    (1, 4 * 128 + 77, 512, 128, True, False, True, True, 1.0),  # HCA ratio, ragged tail
    (2, 300, 128, 16, True, True, False, True, 8.0),      # 16 threads per entry, Za absent, wide logits
    (3, 5, 64, 4, True, False, True, True, 1.0),          # N = 1 (entry 0 only)
    (1, 90, 48, 5, True, True, True, True, 30.0),         # 6 threads per entry (252-thread blocks), sharp softmax
    (1, 40, 2048, 2, True, False, True, True, 1.0),       # 256 threads per entry
    (2, 333, 8, 7, True, False, True, True, 4.0),         # one thread per entry
])
def test_compress_dynamic_parity(cuda, batch, T, d, m, rms, use_gain, za, zb, z_scale):
    A, B, Za, Zb, bias = _dyn_inputs(batch, T, d, m, z_scale)
    Za = Za if za else None
    Zb = Zb if zb else None
    gain = (seeded((d,), 64, "uniform") + 0.5) if use_gain else None
    out = cuda.csa_compress_dynamic(A, B, Za, Zb, bias, m, rms, gain, 1e-6)
    ref = oracle.compress_dynamic(bits(A), bits(B), None if Za is None else bits(Za), None if Zb is None else bits(Zb),
                                  bias.cpu().numpy(), m, rms, None if gain is None else gain.cpu().numpy(), 1e-6)
    _check_rows(f64(out), ref)
    again = cuda.csa_compress_dynamic(A, B, Za, Zb, bias, m, rms, gain, 1e-6)
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))   # fixed reduction order


def test_compress_dynamic_minus_inf_bias_rows_and_no_z(cuda):
    """-inf bias drops a row for the channels it covers; with no Z the call is
    csa_compress on the same logits."""
    batch, T, d, m = 2, 203, 128, 4
    A, B, Za, Zb, bias = _dyn_inputs(batch, T, d, m, seed=70)
    bias[0, : d // 2] = float("-inf")
    bias[2 * m - 1, d // 4:] = float("-inf")
    out = cuda.csa_compress_dynamic(A, B, Za, Zb, bias, m)
    ref = oracle.compress_dynamic(bits(A), bits(B), bits(Za), bits(Zb), bias.cpu().numpy(), m)
    _check_rows(f64(out), ref)
    bias2 = torch.randn((2 * m, d), generator=torch.Generator(DEV).manual_seed(71), device=DEV)
    plain = cuda.csa_compress_dynamic(A, B, None, None, bias2, m)
    _check_rows(f64(plain), oracle.compress(bits(A), bits(B), bias2.cpu().numpy(), m))


def test_compress_dynamic_appends_into_a_cache(cuda):
    """Entries [i0, i0+ni) land in rows i0.. of a longer cache; every other row
    keeps its bits (decode-time compression, one entry every m tokens)."""
    batch, T, d, m = 3, 96, 512, 4
    A, B, Za, Zb, bias = _dyn_inputs(batch, T, d, m, seed=80)
    n_out = 40
    cache = torch.full((batch, n_out, d), 7.0, dtype=torch.bfloat16, device=DEV)
    before = cache.clone()
    for i0, ni in ((0, 1), (5, 3), (T // m - 1, 1)):
        cuda.csa_compress_dynamic(A, B, Za, Zb, bias, m, i0=i0, ni=ni, out=cache)
        ref = oracle.compress_dynamic(bits(A), bits(B), bits(Za), bits(Zb), bias.cpu().numpy(), m, i0=i0, ni=ni)
        _check_rows(f64(cache[:, i0:i0 + ni]), ref)
    written = torch.zeros(n_out, dtype=torch.bool)
    written[[0, 5, 6, 7, T // m - 1]] = True
    assert torch.equal(cache[:, ~written].view(torch.int16), before[:, ~written].view(torch.int16))


def test_compress_dynamic_decode_128k_cache_sampled(cuda):
    """The 128K decode cache (8 x 131072 tokens, d = 512, m = 4) built in one
    launch, checked on sampled entries: entry i depends only on token rows
    (i-1)m .. (i+1)m-1, so the oracle computes it from those rows alone."""
    wl = W.CSA_DECODE
    bsz, T, d, m = wl.batch, wl.T, wl.D, wl.m
    A = torch.stack([W.stream(wl, "A", b, DEV) for b in range(bsz)])
    B = torch.stack([W.stream(wl, "B", b, DEV) for b in range(bsz)])
    Za = torch.stack([W.compression_weights(wl, "Za", b, DEV) for b in range(bsz)])
    Zb = torch.stack([W.compression_weights(wl, "Zb", b, DEV) for b in range(bsz)])
    bias = W.pool_logits(wl, DEV)
    out = cuda.csa_compress_dynamic(A, B, Za, Zb, bias, m)
    N = T // m
    rs = np.random.default_rng(81)
    bn = bias.cpu().numpy()
    for b in range(bsz):
        ents = np.unique(np.concatenate([[0, 1, N - 1], rs.integers(2, N - 1, 29)]))
        for i in ents:
            lo = max(0, (i - 1) * m)
            rows = slice(lo, (i + 1) * m)
            sub = [bits(t[b:b + 1, rows]) for t in (A, B, Za, Zb)]
            ref = oracle.compress_dynamic(*sub, bn, m, i0=0 if i == 0 else 1, ni=1)
            _check_rows(f64(out[b:b + 1, i:i + 1]), ref)
    del A, B, Za, Zb


# ----------------------------------------------------------------------------- index
def _index_case(batch, nq, H_I, d_I, N, m, ts, seed=20):
    qI = seeded((batch, nq, H_I, d_I), seed)
    w = seeded((batch, nq, H_I), seed + 1, "uniform")
    kI = seeded((batch, N, d_I), seed + 2)
    qp = positions(batch, nq, ts)
    return qI, w, kI, qp


def _check_scores(got, ref, rel):
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    fin = np.isfinite(ref)
    for q in np.ndindex(ref.shape[:-1]):
        f = fin[q]
        if f.any():
            scale = np.abs(ref[q][f]).max()
            assert np.abs(got[q][f] - ref[q][f]).max() <= rel * max(scale, 1e-30), q


@pytest.mark.parametrize("batch,nq,H_I,d_I,N,m,ts", [
    (1, 1, 4, 32, 512, 4, [2047]),                              # tiny workload
    (2, 3, 64, 128, 1000, 4, [3999, 1500, 2, 3, 2222, 3998]),     # ragged N, near-zero positions
    (1, 2, 16, 64, 130, 1, [129, 64]),
    (1, 4, 64, 128, 4096 + 33, 4, [16531, 16500, 8000, 3]),
    (2, 1, 8, 256, 300, 2, [599, 100]),
    (1, 9, 64, 128, 2000, 4, [7999 - 3 * i for i in range(9)]),     # query groups of 4 (+1 ragged)
    (3, 5, 4, 32, 700, 4, [2799, 2000, 1000, 10, 3] * 3),          # H_I padded to 16, 5 queries per tile
    (8, 1, 64, 128, 32768, 4, [131071] * 8),                       # CSA decode shape
])
def test_index_parity(cuda, batch, nq, H_I, d_I, N, m, ts):
    qI, w, kI, qp = _index_case(batch, nq, H_I, d_I, N, m, ts)
    got = f64(cuda.csa_index(qI, w, kI, qp, m))
    ref = oracle.index(bits(qI), w.cpu().numpy(), bits(kI), qp.cpu().numpy(), m)
    _check_scores(got, ref, 1e-3)


# ----------------------------------------------------------------------------- top-k
def _check_topk_exact(got, ref, qp, m, N):
    for q in np.ndindex(ref.shape[:-1]):
        g, r = got[q], ref[q]
        nv = oracle.n_visible(int(qp[q]), m, N)
        assert np.sum(g == -1) == np.sum(r == -1) == max(0, len(r) - nv)
        gv = g[g >= 0]
        assert np.all(np.diff(gv) > 0), "indices must be ascending"
        assert np.array_equal(gv, np.sort(r[r >= 0])), q


@pytest.mark.parametrize("batch,nq,N,m,k,ts,levels", [
    (1, 1, 512, 4, 64, [2047], 0),
    (2, 2, 1000, 4, 64, [3999, 100, 20, 3], 0),          # n_vis < k and n_vis = 0/1
    (1, 3, 5000, 1, 1024, [4999, 1023, 3000], 7),        # heavy ties (7 score levels)
    (8, 1, 32768, 4, 1024, [131071] * 8, 0),             # CSA decode shape
    (1, 2, 262144, 4, 1024, [1048575, 900000], 0),       # FP4 decode shape (cluster of 8-16)
    (3, 1, 777, 1, 1024, [776, 500, 1023], 3),
])
def test_topk_exact_on_identical_scores(cuda, batch, nq, N, m, k, ts, levels):
    r = np.random.default_rng(30 + N)
    s = r.standard_normal((batch, nq, N)).astype(np.float32)
    if levels:
        s = np.floor(s * levels / 2).astype(np.float32)
    s[0, 0, :7] = 0.0
    s[0, 0, 7] = -0.0            # signed zero ties with +0
    qp = positions(batch, nq, ts)
    got = cuda.csa_topk(torch.from_numpy(s).to(DEV), qp, m, k).cpu().numpy()
    ref = oracle.topk(s.astype(np.float64), qp.cpu().numpy(), m, k)
    _check_topk_exact(got, ref, qp.cpu().numpy(), m, N)


@pytest.mark.parametrize("batch,nq,N,k,mode", [
    (8, 1, 32768, 1024, "threshold_ties"),   # ties inside the threshold bin (ranked directly)
    (4, 1, 32768, 1024, "crowded_bin"),      # 33..256 keys in the threshold bin (block-wide ranking)
    (2, 1, 65536, 2048, "crowded_bin"),
    (2, 1, 32768, 1024, "outlier"),          # one huge score: linear bins collapse, radix passes
    (2, 1, 4096, 256, "neg_inf"),            # -inf among the visible scores
    (2, 80, 16384, 1024, "normal"),          # one CTA per query (many queries)
    (1, 160, 16384, 1024, "threshold_ties"),
    (2, 1, 32768, 1024, "shifted"),          # scores far from zero (large exponent, narrow range)
])
def test_topk_exact_value_cases(cuda, batch, nq, N, k, mode):
    """Exact top-k (ties -> lower index) on score sets that take each branch of
    the selector: the threshold bin of the value-linear pass ranked directly,
    and the radix passes over the key bits when that bin is large or the range
    is not finite."""
    r = np.random.default_rng(70 + N + nq)
    s = r.standard_normal((batch, nq, N)).astype(np.float32)
    if mode == "threshold_ties":
        for q in np.ndindex(batch, nq):
            kth = np.sort(s[q])[-k]
            s[q][r.choice(N, 6, replace=False)] = kth      # six more copies of the k-th largest score
    elif mode == "crowded_bin":
        for q in np.ndindex(batch, nq):
            kth = np.sort(s[q])[-k]
            pick = r.choice(N, 100, replace=False)
            # distinct scores within 1e-3 of the k-th largest (one value-linear bin spans ~8e-3),
            # every fifth an exact copy of it
            s[q][pick] = (kth + r.uniform(-1e-3, 1e-3, 100)).astype(np.float32)
            s[q][pick[::5]] = kth
    elif mode == "outlier":
        s[:, :, 100] = 1e30
    elif mode == "neg_inf":
        s[:, :, ::7] = -np.inf
    elif mode == "shifted":
        s = (s * 1e-3 + 3000.0).astype(np.float32)
    m = 4
    qp = torch.full((batch, nq), 4 * N - 1, dtype=torch.int32)
    qp[0, 0] = 4 * (N // 2)                             # one query sees half the entries
    qp = qp.to(DEV)
    got = cuda.csa_topk(torch.from_numpy(s).to(DEV), qp, m, k).cpu().numpy()
    ref = oracle.topk(s.astype(np.float64), qp.cpu().numpy(), m, k)
    _check_topk_exact(got, ref, qp.cpu().numpy(), m, N)


def _check_topk_band(got, ref_scores, qp, m, k, N):
    """Set difference only inside the 1e-4 relative band around the k-th oracle score."""
    for q in np.ndindex(ref_scores.shape[:-1]):
        nv = oracle.n_visible(int(qp[q]), m, N)
        s = ref_scores[q][:nv]
        g = got[q]
        gset = set(g[g >= 0].tolist())
        assert len(gset) == min(k, nv)
        if nv <= k:
            assert gset == set(range(nv))
            continue
        sk = np.sort(s)[::-1][k - 1]
        band = 1e-4 * abs(sk)
        oset = set(oracle.topk(ref_scores[q][None, None], np.array([[qp[q]]], np.int32), m, k)[0, 0].tolist())
        for j in gset ^ oset:
            assert abs(s[j] - sk) <= band, (q, j, s[j], sk)


# ----------------------------------------------------------------------------- attention
def _random_selection(batch, nq, k, ts, m, N, seed):
    r = np.random.default_rng(seed)
    idx = np.full((batch, nq, k), -1, np.int32)
    for b in range(batch):
        for q in range(nq):
            nv = oracle.n_visible(ts[b * nq + q], m, N)
            n = min(k, nv)
            idx[b, q, :n] = r.choice(nv, n, replace=False)
            r.shuffle(idx[b, q])
    return idx


@pytest.mark.parametrize("batch,nq,H,D,N,T,k,Wn,m,ts,gain", [
    (1, 1, 8, 64, 512, 2048, 64, 16, 4, [2047], False),                      # tiny workload
    (2, 2, 128, 512, 300, 1200, 100, 128, 4, [1199, 1100, 700, 5], True),    # V4 heads, n_vis < k
    (1, 3, 128, 512, 1024, 4096, 1024, 128, 4, [4095, 2000, 0], False),      # k = 1024, t = 0
    (2, 1, 40, 128, 97, 400, 33, 7, 4, [399, 13], False),                    # ragged heads
    (1, 1, 128, 256, 64, 256, 16, 1, 4, [255], False),                       # W = 1
])
def test_csa_attend_parity(cuda, batch, nq, H, D, N, T, k, Wn, m, ts, gain):
    q = seeded((batch, nq, H, D), 40)
    kv = seeded((batch, N, D), 41)
    win = seeded((batch, T, D), 42)
    qp = positions(batch, nq, ts)
    g = (seeded((D,), 43, "uniform") + 0.5) if gain else None
    idx = _random_selection(batch, nq, k, ts, m, N, 44)
    scale = 1.0 / np.sqrt(D)
    out = cuda.csa_attend(q, kv, torch.from_numpy(idx).to(DEV), win, qp, Wn, scale, 1e-6, g)
    ref = oracle.attend(bits(q), bits(kv), idx, bits(win), qp.cpu().numpy(), Wn, scale, 1e-6,
                        None if g is None else g.cpu().numpy())
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


@pytest.mark.parametrize("batch,nq,H,D,N,T,k,Wn,m", [
    (8, 1, 128, 512, 32768, 131072, 1024, 128, 4),     # CSA decode shape (split keys + combine)
    (1, 200, 128, 512, 2048, 8192, 128, 16, 4),        # many queries per cluster (prefill-like loop)
    (1, 150, 64, 256, 1000, 4000, 200, 32, 4),         # D = 256: one CTA per query, several per SM slot
])
def test_csa_attend_parity_large(cuda, batch, nq, H, D, N, T, k, Wn, m):
    q = seeded((batch, nq, H, D), 45)
    kv = seeded((batch, N, D), 46)
    ts = [T - 1 - (i % 7) * 3 for i in range(batch * nq)]
    qp = positions(batch, nq, ts)
    p0 = T - 64 - Wn
    win = seeded((batch, T - p0, D), 47)
    idx = _random_selection(batch, nq, k, ts, m, N, 48)
    scale = 1.0 / np.sqrt(D)
    out = cuda.csa_attend(q, kv, torch.from_numpy(idx).to(DEV), win, qp, Wn, scale, win_pos0=p0)
    ref = oracle.attend(bits(q), bits(kv), idx, bits(win), qp.cpu().numpy(), Wn, scale, win_pos0=p0)
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


@pytest.mark.parametrize("batch,nq,H,D,N,T,k,Wn,m,ts", [
    (8, 1, 128, 512, 4096, 16384, 1024, 128, 4, [16383] * 8),      # key splits + merge
    (1, 3, 128, 256, 300, 1200, 64, 16, 4, [1199, 700, 5]),        # one split per query
    (2, 1, 40, 128, 97, 400, 33, 7, 4, [399, 13]),                 # ragged heads
])
def test_csa_attend_sinks_parity(cuda, batch, nq, H, D, N, T, k, Wn, m, ts):
    """Per-head sink logits in the softmax denominator (techniques map,
    "Learnable attention sink"), against the oracle on the same selection."""
    q = seeded((batch, nq, H, D), 64)
    kv = seeded((batch, N, D), 65)
    win = seeded((batch, T, D), 66)
    qp = positions(batch, nq, ts)
    idx = _random_selection(batch, nq, k, ts, m, N, 67)
    sinks = (seeded((H,), 68, "uniform") * 6.0 - 3.0).contiguous()
    scale = 1.0 / np.sqrt(D)
    out = cuda.csa_attend(q, kv, torch.from_numpy(idx).to(DEV), win, qp, Wn, scale, sinks=sinks)
    ref = oracle.attend(bits(q), bits(kv), idx, bits(win), qp.cpu().numpy(), Wn, scale,
                        sinks=sinks.cpu().numpy())
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()
    # a sink of -inf is no sink at all
    plain = cuda.csa_attend(q, kv, torch.from_numpy(idx).to(DEV), win, qp, Wn, scale)
    none = cuda.csa_attend(q, kv, torch.from_numpy(idx).to(DEV), win, qp, Wn, scale,
                           sinks=torch.full((H,), float("-inf"), device=DEV))
    assert torch.equal(plain, none)


def test_hca_attend_sinks_parity(cuda):
    batch, H, D, N, m, Wn = 4, 128, 512, 700, 128, 128
    T = N * m
    q = seeded((batch, 1, H, D), 71)
    kv = seeded((batch, N, D), 72)
    win = seeded((batch, Wn, D), 73)
    qp = positions(batch, 1, [T - 1, T - 1, 300 * 128 + 5, 64])
    sinks = (seeded((H,), 74, "uniform") * 6.0 - 3.0).contiguous()
    out = cuda.hca_attend(q, kv, m, win, qp, Wn, D ** -0.5, win_pos0=T - Wn, sinks=sinks)
    ref = oracle.hca_attend(bits(q), bits(kv), m, bits(win), qp.cpu().numpy(), Wn, D ** -0.5, win_pos0=T - Wn,
                            sinks=sinks.cpu().numpy())
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


def _rope_tables(n_pos, base=10000.0):
    """cos / sin [n_pos][32] of angles p * base^(-i/32) (the 64 rotated channels' 32 pairs)."""
    om = base ** (-np.arange(32) / 32.0)
    ang = np.arange(n_pos)[:, None] * om[None, :]
    c = torch.from_numpy(np.cos(ang).astype(np.float32)).to(DEV)
    s = torch.from_numpy(np.sin(ang).astype(np.float32)).to(DEV)
    return c, s


@pytest.mark.parametrize("batch,nq,H,D,N,T,k,Wn,m,ts,sinks", [
    (8, 1, 128, 512, 4096, 16384, 1024, 128, 4, [16383] * 8, False),     # key splits + merge
    (1, 3, 128, 256, 300, 1200, 64, 16, 4, [1199, 700, 5], True),        # one split per query, with sinks
    (2, 1, 40, 128, 97, 400, 33, 7, 4, [399, 13], False),                # ragged heads
    (1, 2, 8, 64, 512, 2048, 64, 16, 4, [2047, 1000], False),            # D = 64: every channel rotates
    (1, 64, 128, 512, 1024, 4096, 64, 32, 4, [4095 - 5 * i for i in range(64)], False),   # single split, bf16 epilogue
])
def test_csa_attend_rope_parity(cuda, batch, nq, H, D, N, T, k, Wn, m, ts, sinks):
    """Partial RoPE (techniques map "Partial RoPE", rope-conjugate output):
    the 64 trailing channels of the normalised query rotate at its position,
    the output gets the conjugate rotation; keys are inputs as they stand."""
    q = seeded((batch, nq, H, D), 90)
    kv = seeded((batch, N, D), 91)
    win = seeded((batch, T, D), 92)
    qp = positions(batch, nq, ts)
    idx = _random_selection(batch, nq, k, ts, m, N, 93)
    sk = (seeded((H,), 94, "uniform") * 6.0 - 3.0).contiguous() if sinks else None
    cos, sin = _rope_tables(T)
    scale = 1.0 / np.sqrt(D)
    out = cuda.csa_attend(q, kv, torch.from_numpy(idx).to(DEV), win, qp, Wn, scale, sinks=sk, rope=(cos, sin))
    ref = oracle.attend(bits(q), bits(kv), idx, bits(win), qp.cpu().numpy(), Wn, scale,
                        sinks=None if sk is None else sk.cpu().numpy(), rope=(cos.cpu().numpy(), sin.cpu().numpy()))
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()
    # the rotation is not a no-op on these inputs
    plain = oracle.attend(bits(q), bits(kv), idx, bits(win), qp.cpu().numpy(), Wn, scale,
                          sinks=None if sk is None else sk.cpu().numpy())
    assert np.abs(plain - ref).max() > 0.05 * np.abs(ref).max()


def test_attend_rope_paths_cover_split_and_single(cuda):
    """The two output paths the rotation lives in: the merge kernel (several key
    splits) and the attention kernel's own bf16 epilogue (one split)."""
    assert cuda.attend_workspace_bytes(8, 1, 128, 512, 1024 + 128) > 0
    assert cuda.attend_workspace_bytes(1, 64, 128, 512, 64 + 32) == 0


def test_attend_rope_outside_the_table_is_unrotated_and_noalloc_agrees(cuda):
    batch, nq, H, D, N, T, k, Wn, m = 2, 1, 128, 512, 600, 2400, 128, 64, 4
    q = seeded((batch, nq, H, D), 95)
    kv = seeded((batch, N, D), 96)
    win = seeded((batch, T, D), 97)
    qp = positions(batch, nq, [2399, 1500])
    idx = torch.from_numpy(_random_selection(batch, nq, k, [2399, 1500], m, N, 98)).to(DEV)
    cos, sin = _rope_tables(2000)            # position 2399 lies outside, 1500 inside
    out = cuda.csa_attend(q, kv, idx, win, qp, Wn, D ** -0.5, rope=(cos, sin))
    plain = cuda.csa_attend(q, kv, idx, win, qp, Wn, D ** -0.5)
    assert torch.equal(out[0], plain[0])
    assert not torch.equal(out[1], plain[1])
    na = cuda.csa_attend_noalloc(q, kv, idx, win, qp, Wn, D ** -0.5, rope=(cos, sin))
    assert torch.equal(na, out)


def test_hca_attend_rope_parity(cuda):
    batch, H, D, N, m, Wn = 4, 128, 512, 700, 128, 128
    T = N * m
    q = seeded((batch, 1, H, D), 99)
    kv = seeded((batch, N, D), 100)
    win = seeded((batch, Wn, D), 101)
    qp = positions(batch, 1, [T - 1, T - 1, 300 * 128 + 5, T - 2])
    cos, sin = _rope_tables(T)
    out = cuda.hca_attend(q, kv, m, win, qp, Wn, D ** -0.5, win_pos0=T - Wn, rope=(cos, sin))
    ref = oracle.hca_attend(bits(q), bits(kv), m, bits(win), qp.cpu().numpy(), Wn, D ** -0.5, win_pos0=T - Wn,
                            rope=(cos.cpu().numpy(), sin.cpu().numpy()))
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


# FP8 KV cache (techniques map, inference quantization): e4m3 codes, power-of-two block scales
def _fp8_inputs(shape, seed):
    x = seeded(shape, seed).float()
    x = x * torch.exp(torch.linspace(-3, 3, shape[-2], device=DEV))[:, None]    # rows of different sizes
    return x.to(torch.bfloat16)


def test_quantize_fp8_kv_bit_exact(cuda):
    x = _fp8_inputs((3, 77, 512), 110)
    x[0, 5, 128:256] = 0.0                                   # an all-zero block
    x[1, 9, :128] = 2.0 ** -30                               # a tiny block
    x[2, 3, 256:384] = -(2.0 ** 100)                         # a huge block
    x[2, 4, 384:] = 1.9921875 * 2.0 ** 127                   # saturates at the exponent ceiling
    codes, exps = cuda.csa_quantize_fp8_kv(x)
    rc, re_ = oracle.quantize_fp8_kv(bits(x), 128)
    assert np.array_equal(exps.cpu().numpy(), re_)
    assert np.array_equal(codes.cpu().numpy(), rc)


def _oracle_fp8(x):
    """oracle codes / exponents of bf16 rows, and the dequantised rows as bf16 bits (exact)."""
    c, e = oracle.quantize_fp8_kv(bits(x), 128)
    dq = oracle.dequantize_fp8_kv(c, e, 128)
    dq_bits = W.bits(torch.from_numpy(dq).to(torch.bfloat16))
    return c, e, dq_bits


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    return t if dtype is None else t.view(dtype)


@pytest.mark.parametrize("batch,nq,H,D,N,T,k,Wn,m,ts", [
    (8, 1, 128, 512, 4096, 16384, 1024, 128, 4, [16383] * 8),          # key splits + merge
    (1, 64, 128, 512, 1024, 4096, 64, 32, 4, [4095 - 5 * i for i in range(64)]),   # one split
    (2, 1, 40, 128, 97, 400, 33, 7, 4, [399, 13]),                     # ragged heads, D = 128
    (1, 3, 128, 256, 300, 1200, 64, 16, 4, [1199, 700, 5]),
    # 400 work items on at most 148 CTAs: a CTA's last tile of one item is expanded
    # while the next item's first tile is copied
    (1, 200, 128, 512, 2048, 8192, 64, 32, 4, [8191 - 7 * i for i in range(200)]),
])
def test_csa_attend_fp8kv_parity(cuda, batch, nq, H, D, N, T, k, Wn, m, ts):
    """The FP8 cache (quantised by the oracle) against the oracle's attention on
    its dequantised rows, and bit for bit against the bf16 kernel on those rows
    (the conversion in the gather is exact, so the MMA operands are the same)."""
    q = seeded((batch, nq, H, D), 111)
    kv = _fp8_inputs((batch, N, D), 112)
    win = _fp8_inputs((batch, T, D), 113)
    qp = positions(batch, nq, ts)
    idx = _random_selection(batch, nq, k, ts, m, N, 114)
    kc, ke, kdq = _oracle_fp8(kv)
    wc, we, wdq = _oracle_fp8(win)
    scale = 1.0 / np.sqrt(D)
    # rows up to e^3 times larger than unit RMS would give logits of several
    # hundred, where the bf16 rounding of the normalised query alone moves the
    # softmax beyond the tolerance; a small query gain keeps the logits in the
    # range the other attention tests use
    g = (seeded((D,), 118, "uniform") * 0.02 + 0.01).contiguous()
    idx_d = torch.from_numpy(idx).to(DEV)
    out = cuda.csa_attend_fp8kv(q, _dev(kc), _dev(ke), idx_d, _dev(wc), _dev(we), qp, Wn, scale, q_gain=g)
    ref = oracle.attend(bits(q), kdq, idx, wdq, qp.cpu().numpy(), Wn, scale, q_gain=g.cpu().numpy())
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()
    bf = cuda.csa_attend(q, _dev(kdq, torch.bfloat16), idx_d, _dev(wdq, torch.bfloat16), qp, Wn, scale, q_gain=g)
    assert torch.equal(out.view(torch.int16), bf.view(torch.int16))


def test_hca_attend_fp8kv_parity(cuda):
    batch, H, D, N, m, Wn = 4, 128, 512, 700, 128, 128
    T = N * m
    q = seeded((batch, 1, H, D), 115)
    kv = _fp8_inputs((batch, N, D), 116)
    win = _fp8_inputs((batch, Wn, D), 117)
    qp = positions(batch, 1, [T - 1, T - 1, 300 * 128 + 5, 64])
    kc, ke, kdq = _oracle_fp8(kv)
    wc, we, wdq = _oracle_fp8(win)
    out = cuda.hca_attend_fp8kv(q, _dev(kc), _dev(ke), m, _dev(wc), _dev(we), qp, Wn, D ** -0.5, win_pos0=T - Wn)
    ref = oracle.hca_attend(bits(q), kdq, m, wdq, qp.cpu().numpy(), Wn, D ** -0.5, win_pos0=T - Wn)
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


def test_attend_running_max_rescale(cuda):
    """Entries whose norms grow along the key order (logit scale 0.01 -> 5) push
    the running max up by more than 2^8 after the first tiles (the O rescale
    path).  Logits stay in the range where bf16 query operands keep the
    softmax weights within tolerance."""
    batch, H, D, N, m, Wn = 2, 128, 512, 640, 4, 8
    T = N * m
    q = seeded((batch, 1, H, D), 55)
    base = seeded((batch, N, D), 56).float()
    grow = torch.logspace(-2.0, float(np.log10(5.0)), N, device=DEV).view(1, N, 1)
    kv = (base * grow).to(torch.bfloat16).contiguous()
    win = seeded((batch, Wn, D), 57)
    qp = positions(batch, 1, [T - 1, T - 1])
    scale = 1.0 / np.sqrt(D)
    out = cuda.hca_attend(q, kv, m, win, qp, Wn, scale, win_pos0=T - Wn)
    ref = oracle.hca_attend(bits(q), bits(kv), m, bits(win), qp.cpu().numpy(), Wn, scale, win_pos0=T - Wn)
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


def test_csa_attend_window_cache_equals_full_stream(cuda):
    """A decode window cache (win_pos0 = t-W+1, W rows) gives the same output as the whole stream."""
    batch, H, D, N, T, k, Wn, m = 2, 128, 512, 256, 1024, 64, 128, 4
    q = seeded((batch, 1, H, D), 50)
    kv = seeded((batch, N, D), 51)
    A = seeded((batch, T, D), 52)
    qp = positions(batch, 1, [T - 1, T - 1])
    idx = torch.from_numpy(_random_selection(batch, 1, k, [T - 1] * 2, m, N, 53)).to(DEV)
    full = cuda.csa_attend(q, kv, idx, A, qp, Wn, D ** -0.5)
    cache = A[:, T - Wn:].contiguous()
    part = cuda.csa_attend(q, kv, idx, cache, qp, Wn, D ** -0.5, win_pos0=T - Wn)
    torch.cuda.synchronize()
    assert torch.equal(full, part)


def test_attend_deterministic_and_writes_every_output(cuda):
    """Twenty decode-shaped calls, each with its split scratch and its output
    pre-filled with NaN, give finite, bit-identical results: every slot read is
    written in the same call, the split merge runs in a fixed order, and no
    wait inside the kernel returns before the work it waits for."""
    batch, H, D, N, T, k, Wn, m = 8, 128, 512, 4096, 16384, 1024, 128, 4
    q = seeded((batch, 1, H, D), 60)
    kv = seeded((batch, N, D), 61)
    win = seeded((batch, Wn, D), 62)
    ts = [T - 1] * batch
    qp = positions(batch, 1, ts)
    idx = torch.from_numpy(_random_selection(batch, 1, k, ts, m, N, 63)).to(DEV)
    nws = cuda.attend_workspace_bytes(batch, 1, H, D, k + Wn)
    assert nws > 0
    first = None
    for _ in range(20):
        ws = torch.full((nws // 4 + 1,), float("nan"), dtype=torch.float32, device=DEV).view(torch.uint8)
        out = torch.full((batch, 1, H, D), float("nan"), dtype=torch.bfloat16, device=DEV)
        cuda.csa_attend(q, kv, idx, win, qp, Wn, D ** -0.5, out=out, workspace=ws, win_pos0=T - Wn)
        assert bool(torch.isfinite(out).all())
        if first is None:
            first = out.clone()
        else:
            assert torch.equal(out, first)
    assert cuda.csa_sync_status() == 0
    ref = oracle.attend(bits(q), bits(kv), idx.cpu().numpy(), bits(win), qp.cpu().numpy(), Wn, D ** -0.5,
                        win_pos0=T - Wn)
    assert np.abs(f64(first) - ref).max() <= 2e-2 * np.abs(ref).max()


@pytest.mark.parametrize("batch,nq,H,D,N,m,T,Wn,ts", [
    (2, 1, 128, 512, 600, 128, 600 * 128, 128, [600 * 128 - 1, 300 * 128 + 5]),
    (1, 2, 8, 64, 512, 4, 2048, 16, [2047, 9]),
    (3, 1, 64, 256, 1000, 4, 4000, 50, [3999, 2, 1234]),
])
def test_hca_attend_parity(cuda, batch, nq, H, D, N, m, T, Wn, ts):
    q = seeded((batch, nq, H, D), 60)
    kv = seeded((batch, N, D), 61)
    qp = positions(batch, nq, ts)
    p0 = max(0, min(ts) - Wn + 1)
    win = seeded((batch, T - p0, D), 62)
    scale = 1.0 / np.sqrt(D)
    out = cuda.hca_attend(q, kv, m, win, qp, Wn, scale, win_pos0=p0)
    ref = oracle.hca_attend(bits(q), bits(kv), m, bits(win), qp.cpu().numpy(), Wn, scale, win_pos0=p0)
    got = f64(out)
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()


# ----------------------------------------------------------------------------- FP4
def test_quantize_fp4_bit_exact(cuda):
    x = seeded((4096, 128), 70).float()
    x[:, 5] *= 8
    x[:, 77] *= 8
    x[0:3, 0:16] = 0                                    # zero blocks
    x[3, 0:16] = 1e-5                                   # scale underflows to e4m3 0
    x[4, 0:16] = torch.linspace(-3e-3, 3e-3, 16)        # subnormal e4m3 scales
    x[5, 16:32] = torch.linspace(-3000, 3000, 16)       # satfinite scale
    x[6, 32:48] = torch.tensor([6, 3, 1.5, 0.75, 0.25, -0.25, -0.75, 5, 2.5, -5, 1.25, 1.75, 3.5, -0.1, 0, -6.])
    xb = x.to(torch.bfloat16).contiguous()
    p, s = cuda.csa_quantize_fp4(xb)
    rp, rs = oracle.quantize_fp4(bits(xb))
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(p.cpu().numpy(), rp)


@pytest.mark.parametrize("batch,nq,H_I,d_I,N,m,ts", [
    (1, 1, 64, 128, 4096, 4, [16383]),
    (2, 2, 16, 64, 777, 4, [3107, 50, 3000, 7]),
    (1, 40, 64, 128, 2048, 4, [8191 - 197 * i for i in range(40)]),   # several query groups per sequence
    (2, 1, 32, 256, 1500, 4, [5999, 2001]),                              # d_I = 256, ragged last tile
    (1, 2, 64, 128, 131072, 4, [524287, 300001]),                        # 128-key tiles, three accumulators, ~7 tiles per CTA
    (1, 1, 64, 128, 200000, 4, [799999]),                                # 256-key tiles, ~5 per CTA, ragged last tile
])
def test_index_fp4_parity(cuda, batch, nq, H_I, d_I, N, m, ts):
    qI, w, kI, qp = _index_case(batch, nq, H_I, d_I, N, m, ts, seed=80)
    q4, q4s = cuda.csa_quantize_fp4(qI)
    k4, k4s = cuda.csa_quantize_fp4(kI)
    got = f64(cuda.csa_index_fp4(q4, q4s, w, k4, k4s, qp, m))
    rq4, rq4s = oracle.quantize_fp4(bits(qI))
    rk4, rk4s = oracle.quantize_fp4(bits(kI))
    ref = oracle.index_fp4(rq4, rq4s, w.cpu().numpy(), rk4, rk4s, qp.cpu().numpy(), m)
    _check_scores(got, ref, 1e-5)


@pytest.mark.parametrize("batch,nq,H_I,d_I,N,kc,k", [
    (2, 1, 64, 128, 8192, 2048, 512),      # decode shape, over-select 4x
    (1, 3, 16, 64, 1000, 300, 100),        # several queries, small
])
def test_rescore_topk_matches_oracle(cuda, batch, nq, H_I, d_I, N, kc, k):
    """FP4 over-selection re-ranked with the bf16 keys.  The candidates are the
    oracle's own FP4 selection; the expected result is the oracle's exact
    bf16-operand scores restricted to those candidates."""
    m = 4
    ts = [N * m - 1 - 5 * i for i in range(batch * nq)]
    qI, w, kI, qp = _index_case(batch, nq, H_I, d_I, N, m, ts, seed=90)
    wn, qpn = w.cpu().numpy(), qp.cpu().numpy()
    rq4, rq4s = oracle.quantize_fp4(bits(qI))
    rk4, rk4s = oracle.quantize_fp4(bits(kI))
    cand = oracle.topk(oracle.index_fp4(rq4, rq4s, wn, rk4, rk4s, qpn, m), qpn, m, kc)
    # ascending entries, -1 slots last (the order csa_topk writes)
    cand = np.where(cand < 0, np.iinfo(np.int32).max, cand)
    cand.sort(axis=-1)
    cand = np.where(cand == np.iinfo(np.int32).max, -1, cand).astype(np.int32)
    got = cuda.csa_rescore_topk(qI, w, kI, torch.from_numpy(cand).to(DEV), k).cpu().numpy()
    S16 = oracle.index(bits(qI), wn, bits(kI), qpn, m)
    masked = np.full_like(S16, -np.inf)
    for q in np.ndindex(cand.shape[:-1]):
        c = cand[q][cand[q] >= 0]
        masked[q][c] = S16[q][c]
    _check_topk_band(got, masked, qpn, m, k, N)
    # every returned entry is one of the candidates, in ascending order
    for q in np.ndindex(cand.shape[:-1]):
        g = got[q][got[q] >= 0]
        assert set(g.tolist()) <= set(cand[q].tolist())
        assert np.all(np.diff(g) > 0)


def test_rescore_topk_with_every_entry_is_plain_topk(cuda):
    """With every entry as a candidate (and -1 slots mixed in) the re-ranking is
    the plain top-k of the bf16-operand scores."""
    batch, nq, H_I, d_I, N, m, k = 2, 1, 64, 128, 3000, 4, 256
    qI, w, kI, qp = _index_case(batch, nq, H_I, d_I, N, m, [N * m - 1] * batch, seed=95)
    cand = np.tile(np.arange(N, dtype=np.int32), (batch, nq, 1))
    cand = np.concatenate([cand, np.full((batch, nq, 77), -1, np.int32)], axis=2)
    got = cuda.csa_rescore_topk(qI, w, kI, torch.from_numpy(cand).to(DEV), k).cpu().numpy()
    ref = oracle.index(bits(qI), w.cpu().numpy(), bits(kI), qp.cpu().numpy(), m)
    _check_topk_band(got, ref, qp.cpu().numpy(), m, k, N)


# ----------------------------------------------------------------------------- failure path
def test_bounded_wait_times_out_and_context_survives(cuda):
    assert cuda.csa_sync_status() == 0
    cuda.csa_set_wait_budget_ns(2_000_000)      # 2 ms
    try:
        cuda.csa_selftest_wait_timeout()
        assert cuda.csa_sync_status() == cuda.CSA_ERR_TIMEOUT
        assert cuda.csa_sync_status() == 0       # read-and-clear
    finally:
        cuda.csa_set_wait_budget_ns(0)
    # the context is still usable
    A = seeded((1, 64, 64), 90)
    out = cuda.csa_compress(A, A, torch.zeros((8, 64), device=DEV), 4)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
