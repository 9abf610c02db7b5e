"""P0 on the GPU: position ids bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from golden_io import all_position_files, load_positions
from gpu_common import positions, q3
from oracle import q3vl_oracle as O
import q3vl_synth as syn

pytestmark = pytest.mark.gpu


def _run(types, grids):
    m = q3()
    tt = torch.tensor(types, dtype=torch.uint8, device="cuda")
    gd = torch.tensor(grids, dtype=torch.int32, device="cuda").reshape(-1, 3) if grids else None
    return m.mrope_positions(tt, gd)


@pytest.mark.parametrize("name", all_position_files())
def test_golden(name):
    types, grids, want, nxt = load_positions(name)
    pos, got_next = _run(types, grids)
    assert pos.cpu().tolist() == want
    assert got_next == nxt


@pytest.mark.parametrize("w", [syn.TINY_FP32, syn.Q2B_LAYER, syn.Q2B_STACK, syn.Q4B_LAYER,
                               syn.Q32B_ENC, syn.Q32B_ENC_1064], ids=lambda w: w.name)
def test_workloads(w):
    pos, ref, nxt, ref_next = positions(w)
    assert np.array_equal(pos.cpu().numpy(), ref)
    assert nxt == ref_next


def test_random_prompts_long():
    # several chunks of the block scan, many grids, adjacent images
    rng = np.random.default_rng(7)
    for trial in range(20):
        types, grids = [], []
        while len(types) < 9000 + 500 * trial:
            types += [0] * int(rng.integers(0, 40))
            if rng.random() < 0.8:
                r, c = int(rng.integers(1, 33)), int(rng.integers(1, 33))
                types += [1] * (r * c)
                grids.append((1, r, c))
        pos, nxt = _run(types, grids)
        ref, ref_next = O.mrope_positions_tokens(types, grids)
        assert np.array_equal(pos.cpu().numpy(), ref)
        assert nxt == ref_next


@pytest.mark.parametrize("types,grids,code", [
    ([0, 1, 1, 0], [(1, 1, 3)], -3),
    ([0, 1, 1, 1], [], -3),
    ([0, 0], [(1, 1, 1)], -3),
    ([1, 1, 0, 1, 1], [(1, 2, 2)], -3),
    ([1, 1], [(2, 1, 1), (1, 1, 1)], -3),   # the 2-frame video takes both tokens
    ([1], [(0, 1, 1)], -3),                 # a grid with no frames
])
def test_mismatch_reported(types, grids, code):
    with pytest.raises(q3().Q3VLError) as e:
        _run(types, grids)
    assert e.value.code == code


def test_random_prompts_with_videos():
    # videos (t frames) mixed with still images and text, several scan chunks
    rng = np.random.default_rng(8)
    for trial in range(12):
        types, grids = [], []
        while len(types) < 6000 + 700 * trial:
            types += [0] * int(rng.integers(0, 30))
            if rng.random() < 0.8:
                t = int(rng.integers(1, 9)) if rng.random() < 0.5 else 1
                r, c = int(rng.integers(1, 17)), int(rng.integers(1, 17))
                types += [1] * (t * r * c)
                grids.append((t, r, c))
        pos, nxt = _run(types, grids)
        ref, ref_next = O.mrope_positions_tokens(types, grids)
        assert np.array_equal(pos.cpu().numpy(), ref)
        assert nxt == ref_next


def test_single_token():
    pos, nxt = _run([0], [])
    assert pos.cpu().tolist() == [[0], [0], [0]] and nxt == 1


@pytest.mark.parametrize("cut", [4, 7, 127, 4095])
def test_run_broken_at_a_thread_warp_or_chunk_boundary(cut):
    # one image of n tokens whose run is broken by a text token at `cut`; the
    # token after it starts a thread's four tokens (7 -> 8), a warp's (127 ->
    # 128) or the next 4096-token chunk (4095 -> 4096)
    n = cut + 9
    types = [1] * cut + [0] + [1] * (n - cut)
    with pytest.raises(q3().Q3VLError) as e:
        _run(types, [(1, 1, n)])
    assert e.value.code == -3


def test_unaligned_token_types():
    # a token-type array that does not start on a 4-byte boundary takes the
    # byte loads; same positions as the oracle
    rng = np.random.default_rng(9)
    types, grids = [], []
    while len(types) < 5000:
        types += [0] * int(rng.integers(0, 20))
        r, c = int(rng.integers(1, 20)), int(rng.integers(1, 20))
        types += [1] * (r * c)
        grids.append((1, r, c))
    buf = torch.zeros(len(types) + 1, dtype=torch.uint8, device="cuda")
    buf[1:] = torch.tensor(types, dtype=torch.uint8, device="cuda")
    tt = buf[1:]
    assert tt.data_ptr() % 4 == 1
    gd = torch.tensor(grids, dtype=torch.int32, device="cuda").reshape(-1, 3)
    pos, nxt = q3().mrope_positions(tt, gd)
    ref, ref_next = O.mrope_positions_tokens(types, grids)
    assert np.array_equal(pos.cpu().numpy(), ref)
    assert nxt == ref_next
