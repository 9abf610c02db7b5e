"""KV cache and one-token decode on the GPU against the oracle.

Tolerances are those of the bf16 layer. Per token, x' must be within rel L2
1e-2 and the update x' - x within 2e-2; the new K/V rows must be within rel
L2 1e-2. The checks are teacher-forced: the oracle's decode reads the GPU's
own cache rows and, in a stack, the GPU's own input to layer l. Each check
therefore covers the arithmetic of one layer.
"""
import numpy as np
import pytest
import torch

from gpu_common import host, layer_on_device, positions, q3, rel_l2
from oracle import q3vl_oracle as O
import q3vl_synth as syn

pytestmark = pytest.mark.gpu
HD = 128


def _text_pos(start, n):
    p = torch.arange(start, start + n, dtype=torch.int32)
    return torch.stack([p, p, p]).cuda().contiguous()


def _fill(m, cfg, packed, kv, lens, seed):
    """Prompt b: lens[b] rows with text positions 0..L-1, prefilled into slot b.
    Returns the per-sequence host rows [L + 1, H] (the last row is the new token)."""
    g = torch.Generator().manual_seed(seed)
    xs = []
    for b, L in enumerate(lens):
        x = torch.randn(L + 1, cfg.hidden, generator=g).to(torch.bfloat16)
        xs.append(x)
        if L > 0:
            xd = x[:L].cuda().clone()
            m.layer_prefill_kv(cfg, packed, xd, _text_pos(0, L), kv, seq=b)
    return xs


def _cache_rows(kv, b, L, nkv):
    return (host(kv.k[b, :L]).reshape(L, nkv, HD), host(kv.v[b, :L]).reshape(L, nkv, HD))


def _check_token(got, want, xin):
    assert np.all(np.isfinite(got))
    assert rel_l2(got, want) <= 1e-2
    assert rel_l2(got - xin, want - xin) <= 2e-2


@pytest.mark.parametrize("w", [
    syn.Q2B_STACK.with_seq(600).with_layers(1),                 # image span, DeepStack slab
    syn.Q4B_LAYER.with_seq(700, images=((100, 8, 12),)),        # QKV bias, 4 heads per group
], ids=lambda w: f"{w.name}-S{w.seq}")
def test_prefill_kv_writes_the_layers_k_and_v(w):
    m = q3()
    cfg = m.config_of(w)
    raw, packed = layer_on_device(w)
    pos, ref_pos, _, _ = positions(w)
    slab = rows = None
    if w.images and w.deepstack_layers:
        slab = syn.deepstack_slabs(w)[0].cuda()
        rows = torch.tensor(syn.image_rows(w), dtype=torch.int32, device="cuda")
    x0 = syn.hidden_input(w).cuda()
    kv = m.KvCache(cfg, n_seq=3, cap=w.seq + 5)
    x1 = x0.clone()
    m.layer_prefill(cfg, packed, x1, pos, slab, rows)
    x2 = x0.clone()
    m.layer_prefill_kv(cfg, packed, x2, pos, kv, seq=1, ds_slab=slab, ds_rows=rows)
    m.check_device()
    assert torch.equal(x1, x2)          # storing the cache changes nothing else
    k, v = O.kv_rows(O.Config.of(w), raw, host(x0), ref_pos)
    kg, vg = _cache_rows(kv, 1, w.seq, w.n_kv_heads)
    assert rel_l2(kg, k) <= 1e-2 and rel_l2(vg, v) <= 1e-2
    assert not kv.k[0].any() and not kv.k[2].any() and not kv.v[1, w.seq:].any()


@pytest.mark.parametrize("w,lens", [
    (syn.Q2B_LAYER, [0, 1, 129, 300]),             # empty cache, one chunk, chunk edges
    (syn.Q4B_LAYER, [5, 256, 1000]),               # QKV bias, 4 query heads per KV head
    (syn.Q2B_LAYER, [3 * b + 1 for b in range(40)]),  # batch of 40 (MMA N = 48)
    (syn.Q32B_ENC, [64, 700]),                     # 8 query heads per KV head, H = 5120
    # batches whose items span several 128-row chunks (merged in registers):
    (syn.Q2B_LAYER, [900 + 3 * b for b in range(16)]),  # 4 splits of ~2 chunks per (b, g)
    (syn.Q2B_LAYER, [400 + b for b in range(64)]),      # 1 split of 4 chunks per (b, g)
    # clusters of 2 splits, each walking ~8 chunks through the 3-stage ring in several passes
    (syn.Q4B_LAYER, [1900 + 37 * b for b in range(9)]),
    # one CTA slot per item, the last split of a (b, g) merging from global memory
    (syn.Q4B_LAYER, [700 + 13 * b for b in range(10)]),
], ids=["2b-b4", "4b-b3", "2b-b40", "32b-b2", "2b-b16-multichunk", "2b-b64-multichunk",
        "4b-b9-cluster2", "4b-b10-ticket"])
def test_layer_decode_matches_oracle(w, lens):
    m = q3()
    cfg = m.config_of(w)
    raw, packed = layer_on_device(w)
    B, cap = len(lens), max(lens) + 8
    kv = m.KvCache(cfg, n_seq=B, cap=cap)
    xs = _fill(m, cfg, packed, kv, lens, seed=11)
    x_new = torch.stack([x[-1] for x in xs])
    xd = x_new.cuda().clone()
    pos = torch.tensor([lens, lens, lens], dtype=torch.int32).cuda()
    seq = torch.arange(B, dtype=torch.int32, device="cuda")
    lt = torch.tensor(lens, dtype=torch.int32, device="cuda")
    m.layer_decode(cfg, packed, xd, pos, kv, seq, lt)
    m.check_device()
    caches = [_cache_rows(kv, b, L, w.n_kv_heads) for b, L in enumerate(lens)]
    want, k_new, v_new = O.layer_decode(O.Config.of(w), raw, host(x_new),
                                        np.array([lens, lens, lens]),
                                        [c[0] for c in caches], [c[1] for c in caches])
    got = host(xd)
    for b, L in enumerate(lens):
        _check_token(got[b], want[b], host(x_new)[b])
        kg, vg = _cache_rows(kv, b, L + 1, w.n_kv_heads)
        assert rel_l2(kg[L], k_new[b]) <= 1e-2 and rel_l2(vg[L], v_new[b]) <= 1e-2, b


@pytest.mark.parametrize("seq_slots", [[2], [3, 0, 5, 1]], ids=["b1-slot2", "b4-scattered"])
def test_decode_reads_and_writes_the_given_cache_slots(seq_slots):
    # tokens mapped to scattered slots of a 6-slot cache; the other slots hold
    # unrelated rows that must not leak into the result or be written
    m = q3()
    w = syn.Q2B_LAYER
    cfg = m.config_of(w)
    raw, packed = layer_on_device(w)
    B, n_seq, cap = len(seq_slots), 6, 400
    kv = m.KvCache(cfg, n_seq=n_seq, cap=cap)
    g = torch.Generator().manual_seed(21)
    lens = [150 + 37 * s for s in range(n_seq)]
    for s in range(n_seq):                        # every slot gets its own prompt
        xp = torch.randn(lens[s], w.hidden, generator=g).to(torch.bfloat16)
        m.layer_prefill_kv(cfg, packed, xp.cuda(), _text_pos(0, lens[s]), kv, seq=s)
    before_k = kv.k.clone()
    x_new = torch.randn(B, w.hidden, generator=g).to(torch.bfloat16)
    my_lens = [lens[s] for s in seq_slots]
    xd = x_new.cuda().clone()
    pos = torch.tensor([my_lens, my_lens, my_lens], dtype=torch.int32).cuda()
    m.layer_decode(cfg, packed, xd, pos, kv, torch.tensor(seq_slots, dtype=torch.int32).cuda(),
                   torch.tensor(my_lens, dtype=torch.int32).cuda())
    m.check_device()
    caches = [_cache_rows(kv, s, lens[s], w.n_kv_heads) for s in seq_slots]
    want, k_new, _ = O.layer_decode(O.Config.of(w), raw, host(x_new), np.array([my_lens] * 3),
                                    [c[0] for c in caches], [c[1] for c in caches])
    got = host(xd)
    for i, s in enumerate(seq_slots):
        _check_token(got[i], want[i], host(x_new)[i])
        assert rel_l2(host(kv.k[s, lens[s]]).reshape(-1, HD), k_new[i]) <= 1e-2
    # only row lens[s] of each used slot changed
    changed = (kv.k != before_k).any(dim=2).nonzero().tolist()
    assert sorted(changed) == sorted([s, lens[s]] for s in seq_slots)


def test_decode_chain_matches_the_prefill_rows():
    # prefill 200 rows into the cache, decode rows 200, 201, 202 one at a time
    # (advancing on the device); each must match the same row of one prefill
    # over all 203 rows
    m = q3()
    w = syn.Q2B_LAYER.with_seq(203)
    cfg = m.config_of(w)
    _, packed = layer_on_device(w)
    x = syn.hidden_input(w)
    full = x.cuda().clone()
    m.layer_prefill(cfg, packed, full, _text_pos(0, 203))
    S0 = 200
    kv = m.KvCache(cfg, n_seq=1, cap=256)
    m.layer_prefill_kv(cfg, packed, x[:S0].cuda().clone(), _text_pos(0, S0), kv)
    pos = _text_pos(S0, 1)
    seq = torch.zeros(1, dtype=torch.int32, device="cuda")
    lt = torch.full((1,), S0, dtype=torch.int32, device="cuda")
    ws = m.decode_workspace(cfg, 1, 256)
    for i in range(3):
        xd = x[S0 + i:S0 + i + 1].cuda().clone()
        m.layer_decode(cfg, packed, xd, pos, kv, seq, lt, ws)
        m.decode_advance(pos, lt)
        assert rel_l2(host(xd)[0], host(full)[S0 + i]) <= 1e-2, i
    m.check_device()
    assert lt.item() == S0 + 3 and pos.cpu().tolist() == [[S0 + 3]] * 3


def test_stack_decode_2b_28_layers_teacher_forced():
    # the 2B stack's prompt (text, a 16x16 image with DeepStack slabs, text)
    # into the caches, then one text token through 1, 2, ..., 28 layers
    m = q3()
    w = syn.Q2B_STACK
    cfg = m.config_of(w)
    pos, _, nxt, _ = positions(w)
    raws, packed = [], []
    for l in range(w.n_layers):
        raw = syn.layer_weights(w, l)
        raws.append(raw)
        packed.append(m.pack_layer(cfg, {k: v.cuda() for k, v in raw.items()}))
    kvs = m.kv_caches(cfg, w.n_layers, n_seq=1, cap=w.seq + 16)
    slabs = [s.cuda() for s in syn.deepstack_slabs(w)]
    rows = torch.tensor(syn.image_rows(w), dtype=torch.int32, device="cuda")
    m.stack_prefill_kv(cfg, packed, syn.hidden_input(w).cuda(), pos, kvs, 0, None, slabs, rows)
    g = torch.Generator().manual_seed(5)
    x_new = torch.randn(1, w.hidden, generator=g).to(torch.bfloat16).cuda()
    pos_new = _text_pos(nxt, 1)
    seq = torch.zeros(1, dtype=torch.int32, device="cuda")
    lt = torch.full((1,), w.seq, dtype=torch.int32, device="cuda")
    ws = m.decode_workspace(cfg, 1, w.seq + 16)
    outs = [x_new]
    for L in range(1, w.n_layers + 1):
        x = x_new.clone()
        m.stack_decode(cfg, packed[:L], x, pos_new, kvs[:L], seq, lt, ws=ws)
        outs.append(x)
    m.check_device()
    ocfg = O.Config.of(w)
    for l in range(w.n_layers):
        kc, vc = _cache_rows(kvs[l], 0, w.seq, w.n_kv_heads)
        want, _, _ = O.layer_decode(ocfg, raws[l], host(outs[l]), np.full((3, 1), nxt), [kc], [vc])
        _check_token(host(outs[l + 1])[0], want[0], host(outs[l])[0])
    gain = syn.final_norm(w)
    y = x_new.clone()
    m.stack_decode(cfg, packed, y, pos_new, kvs, seq, lt, gain.cuda(), ws)
    m.check_device()
    assert rel_l2(host(y), O.rms_norm(host(outs[-1]), host(gain), w.rms_eps)) <= 1e-2


def test_captured_decode_steps_replay_like_eager_steps():
    m = q3()
    w = syn.Q2B_LAYER.with_layers(2)
    cfg = m.config_of(w)
    packed = [layer_on_device(w, l)[1] for l in range(2)]
    lens = [7, 130, 33]
    B, cap = 3, 200
    kvs = m.kv_caches(cfg, 2, n_seq=B, cap=cap)
    g = torch.Generator().manual_seed(3)
    for l in range(2):
        for b, L in enumerate(lens):
            m.layer_prefill_kv(cfg, packed[l],
                               torch.randn(L, w.hidden, generator=g).to(torch.bfloat16).cuda(),
                               _text_pos(0, L), kvs[l], seq=b)
    x_in = torch.randn(B, w.hidden, generator=g).to(torch.bfloat16).cuda()
    seq = torch.arange(B, dtype=torch.int32, device="cuda")
    ws = m.decode_workspace(cfg, B, cap)

    def state():
        return (torch.tensor([lens, lens, lens], dtype=torch.int32).cuda(),
                torch.tensor(lens, dtype=torch.int32).cuda(),
                [(kv.k.clone(), kv.v.clone()) for kv in kvs])

    # eager: three steps
    pos_e, len_e, saved = state()
    x_e = torch.empty_like(x_in)
    for _ in range(3):
        x_e.copy_(x_in)
        m.stack_decode(cfg, packed, x_e, pos_e, kvs, seq, len_e, ws=ws)
        m.decode_advance(pos_e, len_e)
    torch.cuda.synchronize()
    eager_k = [kv.k.clone() for kv in kvs]
    for kv, (k, v) in zip(kvs, saved):
        kv.k.copy_(k)
        kv.v.copy_(v)
    # captured: one step in a graph, replayed three times
    pos_g, len_g, _ = state()
    x_g = torch.empty_like(x_in)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        x_g.copy_(x_in)
        m.stack_decode(cfg, packed, x_g, pos_g, kvs, seq, len_g, ws=ws)
        m.decode_advance(pos_g, len_g)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    m.check_device()
    assert torch.equal(x_g, x_e)
    assert torch.equal(pos_g, pos_e) and torch.equal(len_g, len_e)
    for kv, k in zip(kvs, eager_k):
        assert torch.equal(kv.k, k)
    del graph


def test_decode_argument_errors():
    m = q3()
    w = syn.Q2B_LAYER
    cfg = m.config_of(w)
    _, packed = layer_on_device(w.with_seq(8))
    kv = m.KvCache(cfg, n_seq=2, cap=16)
    x = torch.zeros((2, w.hidden), dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros((3, 2), dtype=torch.int32, device="cuda")
    seq = torch.arange(2, dtype=torch.int32, device="cuda")
    lt = torch.zeros(2, dtype=torch.int32, device="cuda")
    ws = m.decode_workspace(cfg, 2, 16)
    assert m.decode_workspace_bytes(cfg, 0, 16) == 0
    assert m.decode_workspace_bytes(cfg, 257, 16) == 0
    with pytest.raises(m.Q3VLError) as e:
        m.layer_decode(cfg, packed, x, pos, kv, seq, lt, ws[:1024])
    assert e.value.code == -5
    with pytest.raises(m.Q3VLError) as e:          # 17 rows into a 16-row cache
        m.layer_prefill_kv(cfg, packed, torch.zeros((17, w.hidden), dtype=torch.bfloat16,
                                                     device="cuda"), _text_pos(0, 17), kv)
    assert e.value.code == -2
    with pytest.raises(m.Q3VLError) as e:
        m.layer_prefill_kv(cfg, packed, x, _text_pos(0, 2), kv, seq=2)
    assert e.value.code == -2
    f32 = m.config_of(syn.TINY_FP32)
    assert m.decode_workspace_bytes(f32, 1, 16) == 0
    # a length at the capacity is a device-side range error; nothing faults and
    # the next call runs normally
    lt.fill_(16)
    m.layer_decode(cfg, packed, x, pos, kv, seq, lt, ws)
    code, _ = m.device_status()
    assert code == -2
    lt.fill_(0)
    x.zero_()          # the rejected tokens' rows were left unspecified
    m.layer_decode(cfg, packed, x, pos, kv, seq, lt, ws)
    m.check_device()
    assert torch.isfinite(x.float()).all()
