"""Pins of the oracle's KV cache and incremental decode (no GPU).

The pages define a decoded token's output as the last row of the prefill
re-run over prompt + decoded tokens (hf2q ``qwen3vl_text/forward.rs``,
"Why no KV cache yet"), so the cache form is pinned against the prefill
layer (itself pinned in test_oracle_layer.py) and against closed forms in
which the cache contents are arbitrary.
"""
import numpy as np

from oracle import q3vl_oracle as O
import q3vl_synth as syn

HD = 128


def _tiny(seq=24):
    w = syn.TINY_FP32.with_seq(seq)
    return w, O.Config.of(w)


def _weights(w, layer=0):
    return {k: (None if v is None else v.numpy().astype(np.float64))
            for k, v in syn.layer_weights(w, layer).items()}


def _prompt_positions():
    # T T [image 2x3] T T T: an image inside the prompt so that the prompt's
    # positions are not an arange
    tt = [0, 0] + [1] * 6 + [0, 0, 0]
    pos, nxt = O.mrope_positions_tokens(tt, [(1, 2, 3)])
    return tt, pos, nxt


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_text_positions_after_equal_the_token_walk():
    tt, pos, nxt = _prompt_positions()
    # 0 1 | image at 2 advancing by max(2, 3) = 3 | 5 6 7
    assert nxt == 8
    ext, nxt2 = O.mrope_positions_tokens(tt + [0, 0, 0], [(1, 2, 3)])
    assert np.array_equal(O.text_positions_after(nxt, 3), ext[:, len(tt):])
    assert nxt2 == nxt + 3


def test_kv_rows_are_the_layers_k_and_v():
    w, cfg = _tiny(11)
    W = _weights(w)
    x = np.random.default_rng(0).standard_normal((11, cfg.hidden))
    _, pos, _ = _prompt_positions()
    taps = {}
    O.layer(cfg, W, x, pos, taps=taps)
    k, v = O.kv_rows(cfg, W, x, pos)
    assert np.array_equal(k, taps["k"]) and np.array_equal(v, taps["v"])


def test_decode_equals_last_row_of_the_re_run_prefill():
    w, cfg = _tiny()
    W = _weights(w)
    tt, pos, nxt = _prompt_positions()
    S0 = len(tt)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((S0 + 1, cfg.hidden))
    pos_ext = np.concatenate([pos, O.text_positions_after(nxt, 1)], axis=1)
    want = O.layer(cfg, W, x, pos_ext)[S0]
    k, v = O.kv_rows(cfg, W, x[:S0], pos)
    got, kn, vn = O.layer_decode(cfg, W, x[S0:], pos_ext[:, S0:], [k], [v])
    assert _rel(got[0], want) < 1e-13
    # the appended rows are the extended prefill's K/V row
    k2, v2 = O.kv_rows(cfg, W, x, pos_ext)
    assert np.allclose(kn[0], k2[S0], atol=1e-13) and np.allclose(vn[0], v2[S0], atol=1e-13)


def test_batched_decode_with_ragged_caches():
    # three sequences with 0, 4 and 11 cached rows, decoded in one call
    w, cfg = _tiny()
    W = _weights(w)
    rng = np.random.default_rng(2)
    lens = [0, 4, 11]
    xs = [rng.standard_normal((L + 1, cfg.hidden)) for L in lens]
    kc, vc, x_new, pos_new, want = [], [], [], [], []
    for L, x in zip(lens, xs):
        pos = np.tile(np.arange(L + 1) + 3, (3, 1))       # text prompt starting at 3
        k, v = O.kv_rows(cfg, W, x[:L], pos[:, :L])
        kc.append(k)
        vc.append(v)
        x_new.append(x[L])
        pos_new.append(pos[:, L])
        want.append(O.layer(cfg, W, x, pos)[L])
    got, _, _ = O.layer_decode(cfg, W, np.stack(x_new), np.stack(pos_new, axis=1), kc, vc)
    for b in range(3):
        assert _rel(got[b], want[b]) < 1e-13, b


def test_a_chain_of_decodes_equals_the_re_run_prefill():
    w, cfg = _tiny()
    W = _weights(w)
    tt, pos, nxt = _prompt_positions()
    S0, n = len(tt), 4
    rng = np.random.default_rng(3)
    x = rng.standard_normal((S0 + n, cfg.hidden))
    pos_ext = np.concatenate([pos, O.text_positions_after(nxt, n)], axis=1)
    want = O.layer(cfg, W, x, pos_ext)
    k, v = O.kv_rows(cfg, W, x[:S0], pos)
    for i in range(n):
        p = S0 + i
        got, kn, vn = O.layer_decode(cfg, W, x[p:p + 1], pos_ext[:, p:p + 1], [k], [v])
        assert _rel(got[0], want[p]) < 1e-13, i
        k = np.concatenate([k, kn], axis=0)
        v = np.concatenate([v, vn], axis=0)


def test_uniform_attention_over_an_arbitrary_cache():
    # Wq = Wk = 0: every score is 0, so the new row's o is the plain mean of
    # the L cached V rows and its own v. With Wv = Wo = I, unit gains and a
    # zero FFN: x' = x + (sum_j vc_j + x / rms(x)) / (L + 1), for any cache
    # contents (they need not come from a prefill).
    cfg = O.Config(128, 1, 1, 4)
    W = dict(attn_norm=np.ones(128), wq=np.zeros((128, 128)), wk=np.zeros((128, 128)),
             wv=np.eye(128), q_norm=np.ones(HD), k_norm=np.ones(HD), wo=np.eye(128),
             ffn_norm=np.ones(128), wg=np.zeros((4, 128)), wu=np.zeros((4, 128)),
             wd=np.zeros((128, 4)))
    rng = np.random.default_rng(4)
    for L in (0, 1, 7):
        kc = rng.standard_normal((L, 1, HD))
        vc = rng.standard_normal((L, 1, HD))
        x = rng.standard_normal((1, 128))
        got, _, vn = O.layer_decode(cfg, W, x, np.full((3, 1), 50), [kc], [vc])
        xn = x[0] / np.sqrt(np.mean(x[0] ** 2) + 1e-6)
        assert np.allclose(vn[0, 0], xn, atol=1e-14)
        want = x[0] + (vc[:, 0].sum(axis=0) + xn) / (L + 1)
        assert np.allclose(got[0], want, atol=1e-13), L


def test_empty_cache_gives_each_head_its_own_kv_value():
    # L = 0: one key, softmax weight 1, so o of query head h is v of its KV
    # head h div (nh / nkv)
    w, cfg = _tiny()
    W = _weights(w)
    x = np.random.default_rng(5).standard_normal((1, cfg.hidden))
    taps = {}
    O.layer_decode(cfg, W, x, np.full((3, 1), 9), [np.zeros((0, 2, HD))],
                   [np.zeros((0, 2, HD))], taps=taps)
    for h in range(cfg.n_heads):
        assert np.array_equal(taps["o"][0, h], taps["v"][0, O.kv_head(h, 4, 2)])


def test_zero_output_projections_leave_the_token_unchanged():
    w, cfg = _tiny()
    W = _weights(w)
    W["wo"] = W["wo"] * 0
    W["wd"] = W["wd"] * 0
    rng = np.random.default_rng(6)
    x = rng.standard_normal((2, cfg.hidden))
    kc = [rng.standard_normal((3, 2, HD)), rng.standard_normal((5, 2, HD))]
    got, _, _ = O.layer_decode(cfg, W, x, np.full((3, 2), 8), kc, kc)
    assert np.array_equal(got, x)


def test_stack_decode_equals_the_re_run_stack():
    # two layers, an image with DeepStack slabs in the prompt, a final norm;
    # the decoded token is text, so no slab reaches it
    w, cfg = _tiny()
    Ws = [_weights(w, l) for l in range(2)]
    tt, pos, nxt = _prompt_positions()
    S0 = len(tt)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((S0 + 1, cfg.hidden))
    img = np.array([i for i, t in enumerate(tt) if t == 1])
    slabs = [rng.standard_normal((len(img), cfg.hidden)) * 0.1 for _ in range(3)]
    g = 1.0 + 0.1 * rng.standard_normal(cfg.hidden)
    pos_ext = np.concatenate([pos, O.text_positions_after(nxt, 1)], axis=1)
    want = O.stack(cfg, Ws, x, pos_ext, slabs, img, final_norm=g)[S0]
    _, caches = O.stack_prefill_kv(cfg, Ws, x[:S0], pos, slabs, img)
    caches = [([k], [v]) for k, v in caches]
    got, _ = O.stack_decode(cfg, Ws, x[S0:], pos_ext[:, S0:], caches, final_norm=g)
    assert _rel(got[0], want) < 1e-13
    # the prefill half of stack_prefill_kv is the plain stack
    out, _ = O.stack_prefill_kv(cfg, Ws, x[:S0], pos, slabs, img, final_norm=g)
    assert np.array_equal(out, O.stack(cfg, Ws, x[:S0], pos, slabs, img, final_norm=g))


def test_decode_gqa_equals_replicated_kv_heads():
    # a layer with nh = 4 query heads over nkv = 2 KV heads decodes exactly as
    # the same layer with every KV head repeated nh / nkv times (MHA) over an
    # equally repeated cache: query head h reads KV head h div (nh / nkv)
    w, cfg = _tiny()
    W = _weights(w)
    rep = cfg.n_heads // cfg.n_kv_heads
    W_mha = dict(W)
    for name in ("wk", "wv"):
        blocks = W[name].reshape(cfg.n_kv_heads, HD, -1)
        W_mha[name] = np.repeat(blocks, rep, axis=0).reshape(cfg.n_heads * HD, -1)
    cfg_mha = O.Config(cfg.hidden, cfg.n_heads, cfg.n_heads, cfg.intermediate)
    rng = np.random.default_rng(9)
    L = 13
    kc = rng.standard_normal((L, cfg.n_kv_heads, HD))
    vc = rng.standard_normal((L, cfg.n_kv_heads, HD))
    x = rng.standard_normal((1, cfg.hidden))
    pos = np.full((3, 1), 21)
    gqa, _, _ = O.layer_decode(cfg, W, x, pos, [kc], [vc])
    mha, _, _ = O.layer_decode(cfg_mha, W_mha, x, pos, [np.repeat(kc, rep, axis=1)],
                               [np.repeat(vc, rep, axis=1)])
    assert np.allclose(gqa, mha, rtol=1e-13, atol=1e-13)
