"""Pins of the oracle's embedding gather / soft-token splice and LM head (no GPU)."""
import numpy as np
import pytest

from oracle import q3vl_oracle as O


def test_gather_is_row_selection_and_splice_overwrites_only_its_rows():
    # table row v holds v in every column: the gathered row names its token
    V, H = 50, 8
    table = np.repeat(np.arange(V, dtype=np.float64)[:, None], H, axis=1)
    tokens = [7, 3, 3, 49, 0, 12]
    x = O.embed(table, tokens)
    assert (x[:, 0] == tokens).all() and (x == x[:, :1]).all()
    soft = -1.0 - np.arange(2 * H, dtype=np.float64).reshape(2, H)
    y = O.embed(table, tokens, [4, 1], soft)
    assert (y[4] == soft[0]).all() and (y[1] == soft[1]).all()
    keep = [0, 2, 3, 5]
    assert (y[keep] == x[keep]).all()


@pytest.mark.parametrize("tokens,rows,why", [
    ([1, 2, 50], [], "token id past the table"),
    ([1, -1], [], "negative token id"),
    ([1, 2, 3], [3], "row past the prompt"),
    ([1, 2, 3], [1, 1], "overlapping injections"),
    ([], [], "empty prompt"),
])
def test_embed_validation(tokens, rows, why):
    table = np.zeros((50, 4))
    with pytest.raises(O.OracleError):
        O.embed(table, tokens, rows, np.zeros((len(rows), 4)))


def test_lm_head_on_a_scaled_basis_vector():
    # x = c e_k with unit gains: RMSNorm gives sign(c) sqrt(H) e_k (eps -> 0
    # aside), so logits[v] = sign(c) sqrt(H) W[v, k]
    H, V = 16, 30
    cfg = O.Config(H, 1, 1, 128, rms_eps=0.0)
    W = np.random.default_rng(0).standard_normal((V, H))
    for c in (3.0, -0.25):
        x = np.zeros((1, H))
        x[0, 5] = c
        got = O.lm_head(cfg, x, np.ones(H), W)[0]
        assert np.allclose(got, np.sign(c) * np.sqrt(H) * W[:, 5], rtol=1e-14, atol=1e-14)


def test_lm_head_gain_scales_columns_and_tied_equals_untied():
    rng = np.random.default_rng(1)
    H, V = 24, 40
    cfg = O.Config(H, 1, 1, 128)
    x = rng.standard_normal((3, H))
    g = 1.0 + 0.1 * rng.standard_normal(H)
    table = rng.standard_normal((V, H))
    tied = O.lm_head(cfg, x, g, table)
    # the gain can move from the activations into the weight columns
    untied = O.lm_head(cfg, x, np.ones(H), table * g[None, :])
    assert np.allclose(tied, untied, rtol=1e-12, atol=1e-12)
    # rows are independent
    assert np.allclose(O.lm_head(cfg, x[1:2], g, table)[0], tied[1], rtol=1e-13, atol=1e-13)
