"""Pins of the oracle's MQA backward (oracle/mqa_grad.py) against what the
mathematics fixes: central finite differences of the forward (oracle.mqa.attend)
for every gradient, the closed form of a single key, the softmax's invariance
to a shift of every logit (sink included), the output rotation's transpose,
and an entry selected by two queries collecting both queries' gradients."""
import numpy as np
import pytest

from oracle import mqa as omqa, mqa_grad


def _loss(q, keys, scale, dO, sink):
    o, _ = omqa.attend(q, keys, scale, sink)
    return float(np.sum(dO * o))


def _fd(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[i] += eps
        xm[i] -= eps
        g[i] = (f(xp) - f(xm)) / (2 * eps)
    return g


@pytest.mark.parametrize("with_sink", [False, True])
def test_attend_backward_matches_finite_differences(with_sink):
    rng = np.random.default_rng(7 + with_sink)
    H, d, n, scale = 3, 8, 6, 0.4
    q = rng.standard_normal((H, d))
    keys = rng.standard_normal((n, d))
    dO = rng.standard_normal((H, d))
    sink = rng.standard_normal(H) if with_sink else None
    dq, dk, dz, _ = mqa_grad.attend_backward(q, keys, scale, dO, sink)
    assert np.allclose(dq, _fd(lambda x: _loss(x, keys, scale, dO, sink), q), atol=1e-7)
    assert np.allclose(dk, _fd(lambda x: _loss(q, x, scale, dO, sink), keys), atol=1e-7)
    if with_sink:
        assert np.allclose(dz, _fd(lambda x: _loss(q, keys, scale, dO, x), sink), atol=1e-7)
    else:
        assert dz is None


def test_single_key_closed_form():
    """One key, no sink: every weight is 1, o = k for every head, so the
    scores carry no gradient (dq = 0) and dk is the heads' dO summed."""
    rng = np.random.default_rng(1)
    q, k, dO = rng.standard_normal((4, 5)), rng.standard_normal((1, 5)), rng.standard_normal((4, 5))
    dq, dk, _, dS = mqa_grad.attend_backward(q, k, 0.3, dO)
    assert np.allclose(dq, 0.0) and np.allclose(dS, 0.0)
    assert np.allclose(dk[0], dO.sum(0))


def test_logit_shift_invariance():
    """Adding one constant to every score and the sink changes nothing, so the
    gradients of all logits of a head sum to zero: sum_j dS_hj + dz_h = 0."""
    rng = np.random.default_rng(2)
    q, keys = rng.standard_normal((3, 6)), rng.standard_normal((9, 6))
    dO, sink = rng.standard_normal((3, 6)), rng.standard_normal(3)
    _, _, dz, dS = mqa_grad.attend_backward(q, keys, 0.5, dO, sink)
    assert np.allclose(dS.sum(1) + dz, 0.0, atol=1e-12)
    _, _, _, dS0 = mqa_grad.attend_backward(q, keys, 0.5, dO)
    assert np.allclose(dS0.sum(1), 0.0, atol=1e-12)       # no sink: the scores alone


def test_output_rotation_backward_is_the_transpose():
    rng = np.random.default_rng(3)
    H, d, d_rope, p, theta = 4, 16, 8, 1234, 160000.0
    o, g = rng.standard_normal((H, d)), rng.standard_normal((H, d))
    lhs = np.sum(g * omqa.finish_output(o, p, d_rope, theta))
    rhs = np.sum(mqa_grad.output_rotation_backward(g, p, d_rope, theta) * o)
    assert lhs == pytest.approx(rhs, rel=1e-12, abs=1e-12)


def test_sparse_backward_collects_every_query_on_a_shared_entry():
    """Entries 2 and 5 are selected by both queries: their gradient is the
    finite difference of the batch's total loss."""
    rng = np.random.default_rng(4)
    H, d, N, scale = 2, 6, 8, 0.35
    entries = rng.standard_normal((N, d))
    sel = [np.array([2, 5, 7, -1]), np.array([0, 2, 5, -1])]
    win = [rng.standard_normal((3, d)), rng.standard_normal((2, d))]
    qs = rng.standard_normal((2, H, d))
    dOs = rng.standard_normal((2, H, d))
    sink = rng.standard_normal(H)

    def total(ent):
        t = 0.0
        for i in range(2):
            rows = sel[i][sel[i] >= 0]
            t += _loss(qs[i], np.concatenate([ent[rows], win[i]], 0), scale, dOs[i], sink)
        return t
    dq, dent, dwin, dsink = mqa_grad.sparse_backward(qs, sel, entries, win, scale, dOs, sink)
    assert np.allclose(dent, _fd(total, entries), atol=1e-7)
    assert not dent[[1, 3, 4, 6]].any()                  # rows nobody selected
    # the sink's gradient sums over the queries
    ref = sum(mqa_grad.attend_backward(
        qs[i], np.concatenate([entries[sel[i][sel[i] >= 0]], win[i]], 0), scale, dOs[i],
        sink)[2] for i in range(2))
    assert np.allclose(dsink, ref)
