"""Pins of the oracle's MRoPE position builders (no GPU)."""
import numpy as np
import pytest

from golden_io import all_position_files, load_positions
from oracle.q3vl_oracle import OracleError, mrope_positions_spans, mrope_positions_tokens
import q3vl_synth as syn


@pytest.mark.parametrize("name", all_position_files())
def test_hand_computed_grids(name):
    types, grids, want, nxt = load_positions(name)
    pos, got_next = mrope_positions_tokens(types, grids)
    assert pos.tolist() == want
    assert got_next == nxt


def _spans_from(types, grids):
    spans, i, gi = [], 0, 0
    while i < len(types):
        if types[i] == 1:
            _, r, c = grids[gi]
            spans.append((i, r * c, r, c))
            i += r * c
            gi += 1
        else:
            i += 1
    return spans


@pytest.mark.parametrize("name", all_position_files())
def test_span_form_matches_token_form_on_golden(name):
    types, grids, want, _ = load_positions(name)
    if any(g[0] != 1 for g in grids):
        pytest.skip("the span form (cortiq qwen3te.rs) has no frame axis")
    assert mrope_positions_spans(len(types), _spans_from(types, grids)).tolist() == want


def test_video_frames_shift_only_t_and_text_resumes_after_the_longer_side():
    # inferencelayer vision.rs `mrope_positions`: frame f of a (t, h, w) grid
    # is frame 0 shifted by f on the t axis alone; the counter moves by max(h, w)
    rng = np.random.default_rng(11)
    for _ in range(100):
        t, r, c = (int(v) for v in rng.integers(1, 7, size=3))
        lead = int(rng.integers(0, 5))
        types = [0] * lead + [1] * (t * r * c) + [0] * 3
        pos, nxt = mrope_positions_tokens(types, [(t, r, c)])
        still, _ = mrope_positions_tokens([0] * lead + [1] * (r * c), [(1, r, c)])
        for f in range(t):
            blk = pos[:, lead + f * r * c: lead + (f + 1) * r * c]
            assert (blk - still[:, lead:] == np.array([[f], [0], [0]])).all()
        tail = pos[:, lead + t * r * c:]
        assert (tail == lead + max(r, c) + np.arange(3)).all()
        assert nxt == max(lead + t - 1, lead + max(r, c) + 2) + 1


def test_text_only_is_arange():
    # A text-only prompt gives t = h = w = token index (inferencelayer vision.rs,
    # `mrope_positions` doc; cortiq qwen3te.rs module doc).
    pos, nxt = mrope_positions_tokens([0] * 37, [])
    assert (pos == np.arange(37)[None, :]).all()
    assert nxt == 37


def test_random_prompts_two_forms_agree():
    rng = np.random.default_rng(5)
    for _ in range(200):
        types, grids = [], []
        for _ in range(rng.integers(1, 6)):
            types += [0] * int(rng.integers(0, 5))
            if rng.random() < 0.7:
                r, c = int(rng.integers(1, 6)), int(rng.integers(1, 6))
                types += [1] * (r * c)
                grids.append((1, r, c))
        if not types:
            continue
        pos, nxt = mrope_positions_tokens(types, grids)
        sp = mrope_positions_spans(len(types), _spans_from(types, grids))
        assert (pos == sp).all()
        assert nxt == pos.max() + 1


def test_workload_2b_stack_positions():
    w = syn.Q2B_STACK
    pos, nxt = mrope_positions_tokens(syn.token_types(w), syn.grids(w))
    k = np.arange(256)
    assert (pos[:, :100] == np.arange(100)).all()
    assert (pos[0, 100:356] == 100).all()
    assert (pos[1, 100:356] == 100 + k // 16).all()
    assert (pos[2, 100:356] == 100 + k % 16).all()
    assert (pos[:, 356:] == np.arange(116, 1808)).all()
    assert nxt == 1808


def test_workload_4b_positions():
    w = syn.Q4B_LAYER
    pos, _ = mrope_positions_tokens(syn.token_types(w), syn.grids(w))
    k = np.arange(768)
    assert (pos[0, 512:1280] == 512).all()
    assert (pos[1, 512:1280] == 512 + k // 24).all()
    assert (pos[2, 512:1280] == 512 + k % 24).all()
    assert (pos[:, 1280:] == np.arange(544, 3360)).all()


@pytest.mark.parametrize("types,grids", [
    ([0, 1, 1, 0], [(1, 1, 3)]),          # run shorter than its grid
    ([0, 1, 1, 1], []),                   # placeholders but no grid
    ([0, 0], [(1, 1, 1)]),                # grid left over
    ([1, 1], [(2, 1, 1), (1, 1, 1)]),     # the 2-frame video takes both tokens: a grid is left
    ([1], [(0, 1, 1)]),                   # a grid with no frames
])
def test_rejects_mismatch(types, grids):
    with pytest.raises(OracleError):
        mrope_positions_tokens(types, grids)
