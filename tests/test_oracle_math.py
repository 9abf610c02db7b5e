"""Pins of the oracle's MRoPE, RMSNorm and attention against closed forms (no GPU)."""
import numpy as np
import pytest

from oracle import q3vl_oracle as O

THETA = 5e6
HD = 128


def test_slot_counts_24_20_20():
    axes = [O.slot_axis(i) for i in range(64)]
    assert axes.count(0) == 24 and axes.count(1) == 20 and axes.count(2) == 20


def test_slot_rule_examples():
    # every third slot below 60 goes to h (i = 1 mod 3) and w (i = 2 mod 3)
    assert [O.slot_axis(i) for i in (0, 1, 2, 3, 58, 59, 60, 61, 62, 63)] == \
        [0, 1, 2, 0, 1, 2, 0, 0, 0, 0]


def test_unit_vector_rotation_worked_example():
    # e_0 at text position 1: slot 0 has frequency 1, so the pair (0, 64)
    # becomes (cos 1, sin 1).
    x = np.zeros((2, 1, HD))
    x[:, 0, 0] = 1.0
    pos = np.array([[0, 1]] * 3)
    y = O.rope_rotate(x, O.mrope_angles(pos, THETA))
    assert y[0, 0, 0] == 1.0 and y[0, 0, 64] == 0.0
    assert np.isclose(y[1, 0, 0], np.cos(1.0), rtol=0, atol=1e-15)
    assert np.isclose(y[1, 0, 64], np.sin(1.0), rtol=0, atol=1e-15)
    # e_64 rotates the other way: (-sin 1, cos 1)
    x = np.zeros((1, 1, HD))
    x[0, 0, 64] = 1.0
    y = O.rope_rotate(x, O.mrope_angles(np.array([[1]] * 3), THETA))
    assert np.isclose(y[0, 0, 0], -np.sin(1.0)) and np.isclose(y[0, 0, 64], np.cos(1.0))


@pytest.mark.parametrize("slot,axis", [(1, 1), (2, 2), (3, 0), (58, 1), (59, 2), (61, 0), (62, 0)])
def test_slot_reads_its_axis(slot, axis):
    # an image token with distinct t, h, w: slot i rotates by pos[axis] * theta^(-2i/128)
    tpos = np.array([[5], [7], [9]])
    x = np.zeros((1, 1, HD))
    x[0, 0, slot] = 1.0
    y = O.rope_rotate(x, O.mrope_angles(tpos, THETA))
    ang = tpos[axis, 0] * THETA ** (-2.0 * slot / HD)
    assert np.isclose(y[0, 0, slot], np.cos(ang), atol=1e-14)
    assert np.isclose(y[0, 0, slot + 64], np.sin(ang), atol=1e-14)


def test_text_only_mrope_is_1d_rope_complex_form():
    # With t = h = w the slot map is invisible: the rotation equals ordinary
    # 1-D RoPE, written here as multiplication of z_i = x_i + i x_{i+64} by
    # exp(i p f_i).
    rng = np.random.default_rng(0)
    S, nh = 50, 3
    x = rng.standard_normal((S, nh, HD))
    pos = np.tile(np.arange(S) * 3 + 11, (3, 1))
    y = O.rope_rotate(x, O.mrope_angles(pos, THETA))
    p = pos[0][:, None, None].astype(float)
    f = THETA ** (-np.arange(64) / 64.0)
    z = (x[..., :64] + 1j * x[..., 64:]) * np.exp(1j * p * f)
    assert np.allclose(y[..., :64], z.real, atol=1e-12)
    assert np.allclose(y[..., 64:], z.imag, atol=1e-12)


def test_rotation_preserves_pair_norms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((20, 2, HD))
    pos = rng.integers(0, 5000, size=(3, 20))
    y = O.rope_rotate(x, O.mrope_angles(pos, THETA))
    n0 = x[..., :64] ** 2 + x[..., 64:] ** 2
    n1 = y[..., :64] ** 2 + y[..., 64:] ** 2
    assert np.allclose(n0, n1, rtol=1e-12)


def test_text_scores_depend_only_on_offset():
    # q.k after rotation depends on p - j only (shift invariance of text positions)
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, HD))
    k = rng.standard_normal((1, 1, HD))
    def score(p, j):
        qa = O.rope_rotate(q, O.mrope_angles(np.array([[p]] * 3), THETA))
        ka = O.rope_rotate(k, O.mrope_angles(np.array([[j]] * 3), THETA))
        return float((qa * ka).sum())
    assert np.isclose(score(10, 3), score(1010, 1003), rtol=1e-9)
    assert np.isclose(score(7, 7), float((q * k).sum()), rtol=1e-12)


def test_rms_norm_constant_row():
    c, eps = 0.3, 1e-6
    g = np.linspace(0.5, 1.5, 64)
    y = O.rms_norm(np.full((1, 64), c), g, eps)
    assert np.allclose(y[0], c / np.sqrt(c * c + eps) * g, rtol=1e-14)


def test_rms_norm_mean_square_identity():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 300)) * 0.01
    g = 1 + 0.1 * rng.standard_normal(300)
    eps = 1e-6
    y = O.rms_norm(x, g, eps)
    ms = (x ** 2).mean(axis=1)
    assert np.allclose(((y / g) ** 2).mean(axis=1), ms / (ms + eps), rtol=1e-12)


def test_rms_norm_scale_invariant_without_eps():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 128))
    g = rng.standard_normal(128)
    assert np.allclose(O.rms_norm(x, g, 0.0), O.rms_norm(7.5 * x, g, 0.0), rtol=1e-13)


def test_silu_values():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert np.isclose(O.silu(np.array([1.0]))[0], 1.0 / (1.0 + np.exp(-1.0)))
    assert np.isclose(O.silu(np.array([-30.0]))[0], 0.0, atol=1e-11)


def _qkv(S, nh, nkv, seed, hd=HD):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((S, nh, hd)), rng.standard_normal((S, nkv, hd)),
            rng.standard_normal((S, nkv, hd)))


@pytest.mark.parametrize("S,nh,nkv", [(1, 2, 1), (7, 4, 2), (16, 4, 1)])
def test_attention_brute_force(S, nh, nkv):
    q, k, v = _qkv(S, nh, nkv, S)
    assert np.allclose(O.attention(q, k, v), O.attention_pairs(q, k, v), atol=1e-12)


def test_gqa_equals_replicated_kv():
    q, k, v = _qkv(40, 8, 2, 9)
    rep = np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1)
    assert np.allclose(O.attention(q, k, v), O.attention(q, *rep), atol=1e-13)


def test_gqa_head_grouping_consecutive():
    # heads 0..3 share KV head 0 and heads 4..7 share KV head 1
    assert [O.kv_head(h, 8, 2) for h in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]


def test_attention_causal_rows_ignore_future():
    q, k, v = _qkv(30, 2, 1, 10)
    o = O.attention(q, k, v)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[20:] += 5.0
    k2[20:] -= 3.0
    v2[20:] *= -2.0
    o2 = O.attention(q2, k2, v2)
    assert np.array_equal(o[:20], o2[:20])


def test_softmax_rows_sum_to_one():
    q, k, _ = _qkv(33, 2, 1, 11)
    for h in range(2):
        p = O.softmax_rows(q, k, h, 1)
        assert np.all(np.abs(p.sum(axis=1) - 1.0) < 1e-12)
        assert np.all(np.triu(p, 1) == 0.0)


def test_row_zero_attends_to_itself():
    q, k, v = _qkv(9, 4, 2, 12)
    o = O.attention(q, k, v)
    for h in range(4):
        assert np.allclose(o[0, h], v[0, O.kv_head(h, 4, 2)], atol=1e-15)


def test_zero_queries_give_running_mean():
    # q = 0: every allowed key scores 0, so o_p is the mean of v_0..v_p
    _, k, v = _qkv(25, 2, 1, 13)
    q = np.zeros((25, 2, HD))
    o = O.attention(q, k, v)
    cm = np.cumsum(v[:, 0], axis=0) / np.arange(1, 26)[:, None]
    assert np.allclose(o[:, 0], cm, atol=1e-13) and np.allclose(o[:, 1], cm, atol=1e-13)


def test_attention_row_subset_matches_full():
    q, k, v = _qkv(40, 4, 2, 14)
    rows = np.array([0, 5, 39])
    assert np.allclose(O.attention(q, k, v, rows)[rows], O.attention(q, k, v)[rows], atol=1e-14)
