"""Pins of the oracle's composed layer and stack (no GPU).

Each case reduces the layer to something with a closed form, so a dropped
term, a wrong operand or a swapped gate/up would fail one of them.
"""
import numpy as np
import pytest

from oracle import q3vl_oracle as O
import q3vl_synth as syn

HD = 128


def _cfg(H=128, nh=1, nkv=1, I=4):
    return O.Config(H, nh, nkv, I)


def _zeros(cfg, bias=False):
    H, Dq, Dkv, I = cfg.hidden, cfg.n_heads * HD, cfg.n_kv_heads * HD, cfg.intermediate
    W = dict(attn_norm=np.ones(H), wq=np.zeros((Dq, H)), wk=np.zeros((Dkv, H)),
             wv=np.zeros((Dkv, H)), q_norm=np.ones(HD), k_norm=np.ones(HD),
             wo=np.zeros((H, Dq)), ffn_norm=np.ones(H), wg=np.zeros((I, H)),
             wu=np.zeros((I, H)), wd=np.zeros((H, I)))
    if bias:
        W.update(bq=np.zeros(Dq), bk=np.zeros(Dkv), bv=np.zeros(Dkv))
    return W


def _text_pos(S):
    return np.tile(np.arange(S), (3, 1))


def _random_layer(w):
    return syn.layer_weights(w, 0)


def test_zero_output_projections_are_identity():
    w = syn.TINY_FP32.with_seq(20)
    W = _random_layer(w)
    W["wo"] = W["wo"] * 0
    W["wd"] = W["wd"] * 0
    x = syn.hidden_input(w).numpy().astype(np.float64)
    y = O.layer(O.Config.of(w), W, x, _text_pos(20))
    assert np.array_equal(y, x)


def test_uniform_attention_closed_form():
    # Wq = Wk = 0 -> all scores 0 -> o_p = mean_{j<=p} v_j. With Wv = Wo = I,
    # unit gains and a zero FFN: x'_p = x_p + mean_{j<=p} x_j / rms(x_j).
    cfg = _cfg()
    W = _zeros(cfg)
    W["wv"] = np.eye(128)
    W["wo"] = np.eye(128)
    rng = np.random.default_rng(0)
    S = 12
    x = rng.standard_normal((S, 128))
    y = O.layer(cfg, W, x, _text_pos(S))
    for p in range(S):
        acc = np.zeros(128)
        for j in range(p + 1):
            acc += x[j] / np.sqrt(np.mean(x[j] ** 2) + 1e-6)
        assert np.allclose(y[p], x[p] + acc / (p + 1), atol=1e-13)


def test_one_hot_ffn_closed_form():
    # Attention off (Wo = 0). Gate row reads coordinate a, up row reads b, and
    # the down column writes coordinate c: x'_p[c] = x_p[c] + silu(n_a) n_b with
    # n = x_p / rms(x_p). Which projection carries the SiLU is pinned by a != b.
    cfg = _cfg()
    W = _zeros(cfg)
    a, b, c = 3, 70, 11
    W["wg"][0, a] = 1.0
    W["wu"][0, b] = 1.0
    W["wd"][c, 0] = 1.0
    rng = np.random.default_rng(1)
    S = 5
    x = rng.standard_normal((S, 128))
    y = O.layer(cfg, W, x, _text_pos(S))
    for p in range(S):
        n = x[p] / np.sqrt(np.mean(x[p] ** 2) + 1e-6)
        want = x[p].copy()
        want[c] += n[a] / (1 + np.exp(-n[a])) * n[b]
        assert np.allclose(y[p], want, atol=1e-14)


def test_ffn_gain_and_attn_gain_are_plain():
    # A gain of 2 on the FFN norm doubles n (plain w, not 1 + w).
    cfg = _cfg()
    W = _zeros(cfg)
    W["ffn_norm"] = 2 * np.ones(128)
    W["wu"][0, 5] = 1.0
    W["wg"][0, 6] = 1.0
    W["wd"][0, 0] = 1.0
    x = np.random.default_rng(2).standard_normal((1, 128))
    y = O.layer(cfg, W, x, _text_pos(1))
    n = 2 * x[0] / np.sqrt(np.mean(x[0] ** 2) + 1e-6)
    assert np.isclose(y[0, 0] - x[0, 0], n[6] / (1 + np.exp(-n[6])) * n[5], rtol=1e-13)


def test_bias_enters_before_qk_norm():
    # With zero weights the bias alone forms q and k; the per-head norm then
    # makes q_0 = bq / rms(bq) * q_norm at position 0 (no rotation there).
    cfg = _cfg()
    W = _zeros(cfg, bias=True)
    rng = np.random.default_rng(3)
    W["bq"] = rng.standard_normal(128)
    W["bk"] = rng.standard_normal(128)
    W["q_norm"] = 1 + 0.1 * rng.standard_normal(128)
    x = rng.standard_normal((1, 128))
    taps = {}
    O.layer(cfg, W, x, _text_pos(1), taps=taps)
    bq = W["bq"]
    assert np.allclose(taps["q"][0, 0], bq / np.sqrt(np.mean(bq ** 2) + 1e-6) * W["q_norm"],
                       atol=1e-14)


def test_value_bias_shifts_every_output_equally():
    # softmax weights sum to one, so a v bias adds exactly bv to every o row
    cfg = _cfg()
    W = _zeros(cfg, bias=True)
    W["wv"] = np.eye(128)
    W["wo"] = np.eye(128)
    W["bv"] = np.full(128, 0.25)
    x = np.random.default_rng(4).standard_normal((6, 128))
    taps0, taps1 = {}, {}
    O.layer(cfg, {**W, "bv": np.zeros(128)}, x, _text_pos(6), taps=taps0)
    O.layer(cfg, W, x, _text_pos(6), taps=taps1)
    assert np.allclose(taps1["o"] - taps0["o"], 0.25, atol=1e-14)


def test_layer_is_causal_end_to_end():
    w = syn.TINY_FP32.with_seq(24)
    W = _random_layer(w)
    x = syn.hidden_input(w).numpy().astype(np.float64)
    y = O.layer(O.Config.of(w), W, x, _text_pos(24))
    x2 = x.copy()
    x2[17:] += 1.0
    y2 = O.layer(O.Config.of(w), W, x2, _text_pos(24))
    assert np.array_equal(y[:17], y2[:17])
    assert not np.allclose(y[17:], y2[17:])


def test_deepstack_adds_slab_on_image_rows_only():
    w = syn.TINY_FP32.with_seq(16)
    W = _random_layer(w)
    cfg = O.Config.of(w)
    x = syn.hidden_input(w).numpy().astype(np.float64)
    pos = _text_pos(16)
    rows = np.array([3, 4, 5, 9])
    slab = np.random.default_rng(5).standard_normal((4, w.hidden))
    y0 = O.layer(cfg, W, x, pos)
    y1 = O.layer(cfg, W, x, pos, slab, rows)
    d = y1 - y0
    assert np.allclose(d[rows], slab, atol=1e-14)
    mask = np.ones(16, bool)
    mask[rows] = False
    assert np.array_equal(d[mask], np.zeros_like(d[mask]))
    # a zero slab is a no-op
    assert np.array_equal(O.layer(cfg, W, x, pos, np.zeros_like(slab), rows), y0)


def test_deepstack_validation():
    w = syn.TINY_FP32.with_seq(8)
    W = _random_layer(w)
    cfg = O.Config.of(w)
    x = syn.hidden_input(w).numpy().astype(np.float64)
    with pytest.raises(O.OracleError):
        O.layer(cfg, W, x, _text_pos(8), np.zeros((1, w.hidden)), np.array([8]))
    with pytest.raises(O.OracleError):
        O.stack(cfg, [W], x, _text_pos(8), ds_slabs=[np.zeros((1, w.hidden))] * 2,
                ds_rows=np.array([1]))
    with pytest.raises(O.OracleError):
        O.stack(cfg, [W], x, _text_pos(8), ds_slabs=[np.zeros((0, w.hidden))] * 3,
                ds_rows=np.array([], dtype=int))


def test_stack_final_norm_and_slab_order():
    w = syn.TINY_FP32.with_seq(10).with_layers(2)
    cfg = O.Config.of(w)
    Ws = [syn.layer_weights(w, l) for l in range(2)]
    x = syn.hidden_input(w).numpy().astype(np.float64)
    pos = _text_pos(10)
    rows = np.array([2, 3])
    rng = np.random.default_rng(6)
    slabs = [rng.standard_normal((2, w.hidden)) for _ in range(3)]
    g = 1 + 0.1 * rng.standard_normal(w.hidden)
    y = O.stack(cfg, Ws, x, pos, slabs, rows, final_norm=g)
    h = O.layer(cfg, Ws[0], x, pos, slabs[0], rows)
    h = O.layer(cfg, Ws[1], h, pos, slabs[1], rows)
    assert np.array_equal(y, O.rms_norm(h, g, 1e-6))
    # no final norm -> the unnormalised stream
    assert np.array_equal(O.stack(cfg, Ws, x, pos, slabs, rows), h)


def test_row_subset_matches_full_layer():
    w = syn.TINY_FP32.with_seq(40)
    W = _random_layer(w)
    cfg = O.Config.of(w)
    x = syn.hidden_input(w).numpy().astype(np.float64)
    pos = _text_pos(40)
    rows = np.array([0, 13, 39])
    full = O.layer(cfg, W, x, pos)
    sub = O.layer(cfg, W, x, pos, rows=rows)
    assert np.allclose(sub[rows], full[rows], atol=1e-13)
