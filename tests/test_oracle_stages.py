"""Pins of the oracle's method stages against what the pages and the
mathematics fix: closed forms (mean pooling, one-hot gates), textbook
attention (torch SDPA in float64), library routines (scipy softmax /
logsumexp, complex exponentials), invariants (RMS, norms, sums to one,
relative-position property) and brute force on tiny inputs."""
import itertools

import numpy as np
import pytest
import scipy.special
import torch

from oracle import compress, indexer, mqa
from oracle.rope import inv_freq, rmsnorm, rope

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------- RMSNorm / RoPE (I7)

def test_rmsnorm_unit_rms():
    x = RNG.standard_normal((20, 512)) * RNG.uniform(0.1, 10, (20, 1))
    y = rmsnorm(x, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-12)
    assert np.allclose(y / np.linalg.norm(y, axis=-1, keepdims=True),
                       x / np.linalg.norm(x, axis=-1, keepdims=True), atol=1e-12)


def test_rope_matches_complex_rotation():
    d, dr, theta = 128, 32, 160000.0
    x = RNG.standard_normal((9, d))
    pos = RNG.integers(0, 1 << 20, 9)
    y = rope(x, pos, dr, theta)
    z = x[:, d - dr::2] + 1j * x[:, d - dr + 1::2]
    freqs = np.array([theta ** (-(2.0 * i) / dr) for i in range(dr // 2)])
    z = z * np.exp(1j * pos[:, None] * freqs[None, :])
    assert np.allclose(y[:, d - dr::2], z.real, atol=1e-12)
    assert np.allclose(y[:, d - dr + 1::2], z.imag, atol=1e-12)
    assert np.array_equal(y[:, : d - dr], x[:, : d - dr])     # non-RoPE dims untouched


def test_rope_norm_inverse_and_relative_position():
    d, dr, theta = 512, 64, 160000.0
    q = RNG.standard_normal((5, d))
    k = RNG.standard_normal((5, d))
    p = np.array([0, 7, 1000, 65535, 1048575])
    j = np.array([0, 3, 999, 12, 1048000])
    assert np.allclose(np.linalg.norm(rope(q, p, dr, theta), axis=-1), np.linalg.norm(q, axis=-1))
    assert np.allclose(rope(rope(q, p, dr, theta), p, dr, theta, sign=-1.0), q, atol=1e-9)
    lhs = np.sum(rope(q, p, dr, theta) * rope(k, j, dr, theta), axis=-1)
    rhs = np.sum(rope(q, p - j, dr, theta) * k, axis=-1)
    assert np.allclose(lhs, rhs, atol=1e-8)
    assert inv_freq(64, theta)[0] == 1.0 and np.isclose(inv_freq(64, theta)[-1],
                                                         theta ** (-62 / 64))


# ----------------------------------------------------------------- compression (I2, I3)

def _raw(L, c):
    return (RNG.standard_normal((L, c)), RNG.standard_normal((L, c)),
            RNG.standard_normal((L, c)), RNG.standard_normal((L, c)))


@pytest.mark.parametrize("L", [37, 64, 8 * 4 + 3])
def test_csa_uniform_gate_is_mean_pooling(L):
    m, c = 4, 16
    Ca, Za, Cb, Zb = _raw(L, c)
    const = np.zeros((L, c)) + 0.7                      # uniform logits, zero bias
    ii = np.arange(compress.n_entries(L, m))
    e = compress.pool(ii, m, True, L, Ca, const, np.zeros((2 * m, c)), Cb, const)
    for i in ii:
        b_rows = [Cb[t] for t in range(m * (i - 1), m * i) if 0 <= t < L]
        a_rows = [Ca[t] for t in range(m * i, m * (i + 1)) if t < L]
        assert np.allclose(e[i], np.mean(np.array(b_rows + a_rows), axis=0), atol=1e-12)
    assert len(ii) == -(-L // m)


def test_hca_uniform_gate_is_mean_pooling():
    m, c, L = 128, 8, 128 * 3 + 5
    Ca, Za, _, _ = _raw(L, c)
    ii = np.arange(compress.n_entries(L, m))
    e = compress.pool(ii, m, False, L, Ca, np.zeros((L, c)), np.zeros((m, c)))
    for i in ii:
        assert np.allclose(e[i], Ca[m * i: min(L, m * (i + 1))].mean(axis=0), atol=1e-12)


def test_csa_gate_weights_are_a_joint_softmax():
    """One-hot values read the gate weight of each window token; it must be
    scipy's softmax over the 2m logits Z + B (branches sharing one softmax)."""
    m, c, L = 4, 3, 40
    _, Za, _, Zb = _raw(L, c)
    bias = RNG.standard_normal((2 * m, c)) * 0.1
    i = 5
    toks = np.arange(m * (i - 1), m * (i + 1))
    logits = np.concatenate([Zb[toks[:m]], Za[toks[m:]]]) + bias
    want = scipy.special.softmax(logits, axis=0)
    for r, t in enumerate(toks):
        onehot = np.zeros((L, c))
        onehot[t] = 1.0
        Ca = onehot if r >= m else np.zeros((L, c))
        Cb = onehot if r < m else np.zeros((L, c))
        got = compress.pool(np.array([i]), m, True, L, Ca, Za, bias, Cb, Zb)[0]
        assert np.allclose(got, want[r], atol=1e-12), r


def test_csa_bias_and_branch_assignment():
    """A dominant bias at window position r selects exactly token m(i-1)+r,
    read from branch b for r < m and branch a for r >= m."""
    m, c, L = 4, 6, 48
    Ca, Za, Cb, Zb = _raw(L, c)
    for i in (1, 6, 11):
        for r in range(2 * m):
            bias = np.zeros((2 * m, c))
            bias[r] = 200.0
            e = compress.pool(np.array([i]), m, True, L, Ca, Za, bias, Cb, Zb)[0]
            t = m * (i - 1) + r
            assert np.allclose(e, (Ca if r >= m else Cb)[t], atol=1e-9), (i, r)


def test_first_entry_excludes_missing_tokens():
    m, c, L = 4, 5, 20
    Ca, Za, Cb, Zb = _raw(L, c)
    bias = np.zeros((2 * m, c))
    bias[0] = 500.0                                 # would pick token -4 if it existed
    e = compress.pool(np.array([0]), m, True, L, Ca, Za, bias, Cb, Zb)[0]
    w = scipy.special.softmax(Za[0:4], axis=0)
    assert np.allclose(e, np.sum(w * Ca[0:4], axis=0), atol=1e-12)


def test_entry_counts_and_visibility():
    assert compress.n_entries(2 ** 20, 128) == 8192
    assert compress.n_entries(10 ** 6, 128) == 7813
    assert compress.n_entries(2 ** 20, 4) == 262144
    assert compress.n_entries(131072, 4) == 32768 and compress.n_entries(131072, 128) == 1024
    assert compress.n_entries(8192, 4) == 2048
    # R3: the block of the query is invisible until its last token
    assert compress.n_visible(3, 4) == 1 and compress.n_visible(2, 4) == 0
    assert compress.n_visible(131071, 128) == 1024 and compress.n_visible(131070, 128) == 1023


def test_finish_main_norm_then_rope():
    e = RNG.standard_normal((3, 64))
    out = compress.finish_main(e, np.array([0, 1, 2]), 4, 16, 160000.0, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(out * out, axis=-1)), 1.0)   # RoPE keeps the norm
    assert np.allclose(out[0], rmsnorm(e[0], 0.0))                   # position 0: no rotation


# ----------------------------------------------------------------- indexer / top-k

def test_indexer_single_head_onehot_query():
    keys = RNG.standard_normal((30, 128))
    for h, dim in ((0, 5), (3, 127), (63, 64)):
        qI = np.zeros((64, 128))
        qI[h, dim] = 1.0
        w = np.zeros(64)
        w[h] = 1.0
        assert np.allclose(indexer.scores(qI, w, keys), np.maximum(keys[:, dim], 0))


def test_indexer_relu_identity_and_homogeneity():
    qI = RNG.standard_normal((8, 32))
    w = RNG.uniform(0, 1, 8)
    keys = RNG.standard_normal((50, 32))
    s_pos = indexer.scores(qI, w, keys)
    s_neg = indexer.scores(-qI, w, keys)
    assert np.allclose(s_pos + s_neg, np.abs(keys @ qI.T) @ w)       # relu(x)+relu(-x)=|x|
    assert np.allclose(s_pos - s_neg, (keys @ qI.T) @ w)             # relu(x)-relu(-x)=x
    assert np.allclose(indexer.scores(2.5 * qI, w, keys), 2.5 * s_pos)
    w2 = RNG.uniform(0, 1, 8)
    assert np.allclose(indexer.scores(qI, w + w2, keys), s_pos + indexer.scores(qI, w2, keys))


def test_topk_equals_brute_force_with_ties():
    for trial in range(40):
        n = int(RNG.integers(1, 10))
        k = int(RNG.integers(1, 7))
        s = RNG.integers(0, 4, n).astype(np.float64)               # forced exact ties
        n_vis = int(RNG.integers(0, n + 1))
        got = indexer.topk(s, n_vis, k)
        kk = min(k, n_vis)
        # brute force: the unique subset whose worst key (-s, i) beats every outsider
        best = None
        for sub in itertools.combinations(range(n_vis), kk):
            inside = [(-s[i], i) for i in sub]
            outside = [(-s[i], i) for i in range(n_vis) if i not in sub]
            if not outside or max(inside) < min(outside):
                assert best is None
                best = sub
        assert best is not None
        want = list(best) + [-1] * (k - kk)
        assert list(got) == want, (s, n_vis, k, got, want)


# ----------------------------------------------------------------- MQA (I1, I4, I8)

def _sdpa(q, K):
    qt = torch.from_numpy(q)[None, :, None, :]        # [1, H, 1, d]
    kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], K.shape[0], K.shape[1])
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, kt)[0, :, 0].numpy()


def test_degenerate_method_is_causal_mqa():
    """I1: m = 1, no overlap, no norm/RoPE, n_win = 0, top-k = all, no sink is
    plain causal single-KV-head attention with K = V (torch SDPA, float64)."""
    L, d, H = 40, 32, 4
    C = RNG.standard_normal((L, d))
    Z = RNG.standard_normal((L, d))
    ents = compress.pool(np.arange(L), 1, False, L, C, Z, np.zeros((1, d)))
    assert np.allclose(ents, C, atol=1e-15)
    for p in (0, 1, 17, L - 1):
        nv = int(compress.n_visible(p, 1))
        q = RNG.standard_normal((H, d))
        s = indexer.scores(RNG.standard_normal((2, d)), np.ones(2), ents[:nv])
        idx = indexer.topk(s, nv, L)
        keys = ents[np.sort(idx[idx >= 0])]
        o, _ = mqa.attend(q, keys, 1.0 / np.sqrt(d), None)
        assert np.allclose(o, _sdpa(q, C[: p + 1]), atol=1e-12)


def test_sink_limits_and_total_weight():
    H, n, d = 6, 20, 16
    q = RNG.standard_normal((H, d))
    K = RNG.standard_normal((n, d))
    sink = RNG.standard_normal(H)
    o, lse, a, share = mqa.attend(q, K, 0.3, sink, return_weights=True)
    assert np.allclose(a.sum(axis=1) + share, 1.0, atol=1e-12)      # I4
    s = 0.3 * q @ K.T
    assert np.allclose(share, 1.0 / (1.0 + np.exp(s - sink[:, None]).sum(axis=1)), atol=1e-12)
    assert np.allclose(lse, scipy.special.logsumexp(np.concatenate([s, sink[:, None]], 1), axis=1))
    o_hi, _ = mqa.attend(q, K, 0.3, np.full(H, 1e4))                 # I8: sink -> +inf
    assert np.max(np.abs(o_hi)) < 1e-300
    o_lo, _ = mqa.attend(q, K, 0.3, np.full(H, -1e4))                # I8: sink -> -inf
    o_no, _ = mqa.attend(q, K, 0.3, None)
    assert np.allclose(o_lo, o_no, atol=1e-14)
    assert np.allclose(o_no, _sdpa(q * 0.3 * np.sqrt(d), K), atol=1e-12)


def test_output_is_in_span_of_keys():
    q = RNG.standard_normal((4, 64))
    K = RNG.standard_normal((3, 64))
    o, _ = mqa.attend(q, K, 0.125, RNG.standard_normal(4))
    coef, *_ = np.linalg.lstsq(K.T, o.T, rcond=None)
    assert np.allclose(K.T @ coef, o.T, atol=1e-10)


def test_inverse_rope_recovers_unrotated_value():
    """One key k = R(p) u attended alone (no sink) gives o = k; rotating the
    output back by -p returns u exactly (R7)."""
    d, dr, theta, p = 512, 64, 160000.0, 123457
    u = RNG.standard_normal((1, d))
    k = rope(u, np.array([p]), dr, theta)
    o, _ = mqa.attend(RNG.standard_normal((2, d)), k, 0.04, None)
    assert np.allclose(mqa.finish_output(o, p, dr, theta), np.repeat(u, 2, 0), atol=1e-9)


def test_window_tokens():
    assert list(mqa.window_tokens(5, 128)) == list(range(0, 6))
    w = mqa.window_tokens(1000, 128)
    assert w[0] == 873 and w[-1] == 1000 and len(w) == 128
    assert len(mqa.window_tokens(1000, 0)) == 0
