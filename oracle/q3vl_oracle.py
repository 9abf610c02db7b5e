"""CPU oracle for the Qwen3-VL text-decoder causal prefill.

TEST INFRASTRUCTURE ONLY. This module is a plain, slow, obviously correct
statement of what the prefill computes. Only the tests, the smoke check and
the benchmark's CPU-baseline leg may import it; the library never calls it,
and it shares no code, table or helper with the CUDA path.

Everything runs in float64 (``dtype=np.float64``) for parity; ``np.float32``
gives the same algorithm in single precision for the CPU timing baseline.
Inputs given in bf16 are consumed as their exact values, upcast.

Sources (the pages' own items; the pages print Rust, restated here):

* cortiq-engine ``qwen3te.rs`` -- the Qwen3-VL prompt encoder's host forward:
  ``rms_norm_into``, ``silu``, ``Qwen3Encoder::norm_rope`` (per-head RMSNorm
  then interleaved MRoPE), ``Qwen3Encoder::mrope_positions`` (span form),
  ``Qwen3Encoder::encode_with_images`` (layer order, DeepStack, final norm)
  and the per-pair attention loop / ``Qwen3Encoder::attention_gemm``.
* inferencelayer ``vision.rs`` -- ``mrope_positions`` (token form: runs of
  image placeholders against a grid list, ``next`` position).
* hf2q ``qwen3vl_text/forward.rs`` -- the module doc's per-layer order (bias
  before the q/k norm), the DeepStack contract and input validation of
  ``forward_text_prefill_logits_last``, and "Why no KV cache yet" (a decoded
  token is the last row of the prefill re-run over prompt + decoded tokens),
  which defines the incremental decode at the end of this module; and the
  same function's step 1 (token embedding lookup and soft-token splice) and
  step 4 (final norm and LM head, tied or untied).

Parity status: every function here is pinned by the ``-m "not gpu"`` tests
(hand-computed grids, closed forms, brute force, invariants). The composed
random-weight layer is pinned through its parts and through closed-form
special cases (zero projections, uniform attention, one-hot FFN); the pages
print no numeric output of a full layer, so that composition has no external
numeric pin. The decode functions are pinned against that prefill layer
(the last row of a re-run prefill) and against closed forms that hold for
arbitrary cache contents. The embedding gather and LM head are pinned by
closed forms (coded table rows, a scaled basis vector).
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

HEAD_DIM = 128


class OracleError(ValueError):
    """An input the method rejects (grid/run mismatch, bad DeepStack, ...)."""


# ---------------------------------------------------------------------------
# Positions
# ---------------------------------------------------------------------------

def mrope_positions_tokens(token_types: Sequence[int],
                           grids: Sequence[Tuple[int, int, int]]):
    """3-axis (t, h, w) positions from per-token types, walking the prompt.

    inferencelayer ``vision.rs``, ``mrope_positions``: a text token takes
    (cur, cur, cur) and advances cur by one. An image placeholder starts the
    next grid (t, rows, cols) of merged tokens, t frames of rows x cols (t = 1
    for a still image); its tokens follow the meshgrid of (frame, row, col) in
    'ij' order, token (f, r, c) taking (cur + f, cur + r, cur + c), and the
    whole grid advances cur by max(rows, cols) -- neither its token count nor
    its frame count. Grids are consumed whole and in order, so two adjacent
    images need no text between them. ``next`` is one past the largest
    position on any axis (with t > max(rows, cols) frames that is on the t
    axis, beyond where the following text resumes).

    Returns (pos int64 [3, S], next).
    """
    S = len(token_types)
    pos = np.zeros((3, S), dtype=np.int64)
    cur = 0
    gi = 0
    i = 0
    while i < S:
        if token_types[i] == 0:
            pos[:, i] = cur
            cur += 1
            i += 1
            continue
        if gi >= len(grids):
            raise OracleError("more image placeholders than grids")
        t, rows, cols = grids[gi]
        gi += 1
        if t < 1 or rows < 1 or cols < 1:
            raise OracleError("grid sizes must be >= 1")
        n = t * rows * cols
        if i + n > S or any(token_types[j] != 1 for j in range(i, i + n)):
            raise OracleError("image placeholder run shorter than its grid")
        k = 0
        for f in range(t):
            for r in range(rows):
                for c in range(cols):
                    pos[:, i + k] = (cur + f, cur + r, cur + c)
                    k += 1
        cur += max(rows, cols)
        i += n
    if gi != len(grids):
        raise OracleError("grids left over after the last placeholder")
    nxt = int(pos.max()) + 1 if S else 0
    return pos, nxt


def mrope_positions_spans(S: int, spans: Sequence[Tuple[int, int, int, int]]):
    """The same positions from a span list (start, len, rows, cols).

    cortiq-engine ``qwen3te.rs``, ``Qwen3Encoder::mrope_positions``: every
    token starts at (i, i, i); each span pins t at base = start + offset, lays
    the grid on h/w from base, re-numbers every later token from
    start + max(rows, cols) + offset, and the running offset grows by
    max(rows, cols) - len.
    """
    pos = np.tile(np.arange(S, dtype=np.int64), (3, 1))
    offset = 0
    for start, ln, rows, cols in spans:
        if ln != rows * cols:
            raise OracleError("span length differs from its grid")
        end = start + ln
        base = start + offset
        for i in range(start, end):
            k = i - start
            pos[:, i] = (base, base + k // cols, base + k % cols)
        nxt = start + max(rows, cols)
        for j in range(end, S):
            pos[:, j] = nxt + offset + (j - end)
        offset += max(rows, cols) - ln
    return pos


# ---------------------------------------------------------------------------
# Interleaved MRoPE
# ---------------------------------------------------------------------------

def slot_axis(i: int, sections=(24, 20, 20)) -> int:
    """Axis (0 = t, 1 = h, 2 = w) that frequency slot i (0 <= i < hd/2) reads.

    cortiq-engine ``qwen3te.rs``, ``Qwen3Encoder::norm_rope``: h takes the
    slots i = 1 (mod 3) and w the slots i = 2 (mod 3), each below 3 x its
    section (60 for [24, 20, 20]); every other slot reads t.
    """
    if i % 3 == 1 and i < 3 * sections[1]:
        return 1
    if i % 3 == 2 and i < 3 * sections[2]:
        return 2
    return 0


def mrope_angles(pos: np.ndarray, theta: float, hd: int = HEAD_DIM,
                 sections=(24, 20, 20)) -> np.ndarray:
    """Rotation angle of slot i at token p: pos[axis(i), p] * theta^(-2i/hd).

    Returned as float64 [S, hd/2]. The pages form this angle in f32; here it
    is exact to float64.
    """
    half = hd // 2
    S = pos.shape[1]
    ang = np.empty((S, half), dtype=np.float64)
    for i in range(half):
        freq = float(theta) ** (-2.0 * i / hd)
        ang[:, i] = pos[slot_axis(i, sections)].astype(np.float64) * freq
    return ang


def rope_rotate(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Split-half rotation of every head: pairs (i, i + hd/2).

    x: [S, heads, hd]. x'_i = x_i cos - x_{i+hd/2} sin and
    x'_{i+hd/2} = x_i sin + x_{i+hd/2} cos (``Qwen3Encoder::norm_rope``).
    """
    half = x.shape[-1] // 2
    c = np.cos(angles)[:, None, :].astype(x.dtype)
    s = np.sin(angles)[:, None, :].astype(x.dtype)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


# ---------------------------------------------------------------------------
# Norms and activations
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * g over the last axis.

    cortiq-engine ``qwen3te.rs``, ``rms_norm_into``: a plain gain g (not
    1 + g); the mean of squares is taken in float64 on the pages.
    """
    x64 = x.astype(np.float64)
    ms = np.mean(x64 * x64, axis=-1, keepdims=True)
    inv = 1.0 / np.sqrt(ms + eps)
    return (x64 * inv).astype(x.dtype) * g.astype(x.dtype)


def silu(v: np.ndarray) -> np.ndarray:
    """silu(v) = v / (1 + exp(-v)) (``qwen3te.rs``, ``silu``)."""
    return v / (1.0 + np.exp(-v))


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def kv_head(h: int, n_heads: int, n_kv_heads: int) -> int:
    """Query head h reads KV head h div (n_heads / n_kv_heads)."""
    return h // (n_heads // n_kv_heads)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
              rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Causal GQA attention, one head at a time as two matrix products.

    q [S, nh, hd], k/v [S, nkv, hd] -> o [S, nh, hd]. Row p of head h is
    sum_{j <= p} softmax_j(q_p . k_j / sqrt(hd)) v_j, the row maximum
    subtracted before the exponent (``Qwen3Encoder::attention_gemm``).
    ``rows`` restricts the output to those query rows (others are zero).
    """
    S, nh, hd = q.shape
    nkv = k.shape[1]
    scale = 1.0 / np.sqrt(hd)
    rows = np.arange(S) if rows is None else np.asarray(rows)
    o = np.zeros_like(q)
    mask = np.arange(S)[None, :] > rows[:, None]          # future keys
    for h in range(nh):
        kv = kv_head(h, nh, nkv)
        sc = (q[rows, h, :] @ k[:, kv, :].T) * scale
        sc = np.where(mask, -np.inf, sc)
        sc = sc - sc.max(axis=1, keepdims=True)
        p = np.exp(sc)
        p = p / p.sum(axis=1, keepdims=True)
        o[rows, h, :] = p @ v[:, kv, :]
    return o


def attention_pairs(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """The same attention as scalar loops over (head, query, key) triples.

    The pages' exact small-prompt path (``encode_with_images``' per-pair
    loop). Pure Python; for S <= 16 only.
    """
    S, nh, hd = q.shape
    nkv = k.shape[1]
    scale = 1.0 / np.sqrt(hd)
    o = np.zeros_like(q)
    for h in range(nh):
        kv = kv_head(h, nh, nkv)
        for p in range(S):
            sc = [sum(q[p, h, d] * k[j, kv, d] for d in range(hd)) * scale
                  for j in range(p + 1)]
            mx = max(sc)
            e = [np.exp(s - mx) for s in sc]
            den = sum(e)
            for j in range(p + 1):
                for d in range(hd):
                    o[p, h, d] += e[j] / den * v[j, kv, d]
    return o


def softmax_rows(q: np.ndarray, k: np.ndarray, h: int, n_kv_heads: int) -> np.ndarray:
    """The causal probability matrix of head h ([S, S], zero above the diagonal)."""
    S, nh, hd = q.shape
    kv = kv_head(h, nh, n_kv_heads)
    sc = (q[:, h, :] @ k[:, kv, :].T) / np.sqrt(hd)
    sc = np.where(np.triu(np.ones((S, S), dtype=bool), 1), -np.inf, sc)
    sc = sc - sc.max(axis=1, keepdims=True)
    p = np.exp(sc)
    return p / p.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# Layer and stack
# ---------------------------------------------------------------------------

class Config:
    """Shape and constants of one decoder layer."""

    def __init__(self, hidden, n_heads, n_kv_heads, intermediate, head_dim=HEAD_DIM,
                 rope_theta=5e6, rms_eps=1e-6, mrope_section=(24, 20, 20)):
        self.hidden = hidden
        self.n_heads = n_heads
        self.n_kv_heads = n_kv_heads
        self.intermediate = intermediate
        self.head_dim = head_dim
        self.rope_theta = rope_theta
        self.rms_eps = rms_eps
        self.mrope_section = tuple(mrope_section)

    @classmethod
    def of(cls, w) -> "Config":
        return cls(w.hidden, w.n_heads, w.n_kv_heads, w.intermediate, w.head_dim,
                   w.rope_theta, w.rms_eps, w.mrope_section)


def _np(t, dtype):
    if t is None:
        return None
    if hasattr(t, "detach"):                      # a torch tensor
        t = t.detach().to("cpu")
        t = t.float() if str(t.dtype) == "torch.bfloat16" else t
        t = t.numpy()
    return np.asarray(t, dtype=dtype)


def qkv(cfg: Config, W: Dict, x: np.ndarray, angles: np.ndarray, dtype=np.float64,
        q_rows: Optional[np.ndarray] = None):
    """Steps up to the attention inputs: norm, projections (+bias), q/k norm, MRoPE.

    Returns q [S, nh, hd], k [S, nkv, hd], v [S, nkv, hd]. The bias is added
    right after the projection and before the per-head norm (hf2q
    ``qwen3vl_text/forward.rs`` module doc); the per-head norm comes before
    the rotation (``Qwen3Encoder::norm_rope``). With ``q_rows`` only those
    rows of q are formed (the others stay zero); k and v always cover every row.
    """
    S = x.shape[0]
    hd, nh, nkv = cfg.head_dim, cfg.n_heads, cfg.n_kv_heads
    qr = np.arange(S) if q_rows is None else np.asarray(q_rows)
    xn = rms_norm(x, _np(W["attn_norm"], dtype), cfg.rms_eps)
    q = xn[qr] @ _np(W["wq"], dtype).T
    k = xn @ _np(W["wk"], dtype).T
    v = xn @ _np(W["wv"], dtype).T
    if W.get("bq") is not None:
        q = q + _np(W["bq"], dtype)
        k = k + _np(W["bk"], dtype)
        v = v + _np(W["bv"], dtype)
    q = rms_norm(q.reshape(len(qr), nh, hd), _np(W["q_norm"], dtype), cfg.rms_eps)
    k = rms_norm(k.reshape(S, nkv, hd), _np(W["k_norm"], dtype), cfg.rms_eps)
    q_all = np.zeros((S, nh, hd), dtype=q.dtype)
    q_all[qr] = rope_rotate(q, angles[qr])
    return q_all, rope_rotate(k, angles), v.reshape(S, nkv, hd)


def o_residual(W: Dict, o: np.ndarray, x: np.ndarray, dtype=np.float64) -> np.ndarray:
    """h = x + o W_o^T: the o-projection and the attention residual (o: [S, nh*hd])."""
    return x + o @ _np(W["wo"], dtype).T


def ffn_act(cfg: Config, W: Dict, h: np.ndarray, dtype=np.float64) -> np.ndarray:
    """a = silu(hn W_g^T) * (hn W_u^T), hn = RMSNorm(h, ffn_norm)."""
    hn = rms_norm(h, _np(W["ffn_norm"], dtype), cfg.rms_eps)
    return silu(hn @ _np(W["wg"], dtype).T) * (hn @ _np(W["wu"], dtype).T)


def down_residual(W: Dict, a: np.ndarray, h: np.ndarray, dtype=np.float64) -> np.ndarray:
    """x' = h + a W_down^T (before any DeepStack add)."""
    return h + a @ _np(W["wd"], dtype).T


def layer(cfg: Config, W: Dict, x, pos: np.ndarray, ds_slab=None, ds_rows=None,
          dtype=np.float64, rows: Optional[np.ndarray] = None,
          taps: Optional[Dict] = None) -> np.ndarray:
    """One decoder layer x -> x' (``Qwen3Encoder::encode_with_images``' loop body).

    x' = h + W_down(silu(W_gate hn) * W_up hn), hn = RMSNorm(h),
    h = x + W_o attention(MRoPE(norm(q)), MRoPE(norm(k)), v), and for a
    DeepStack layer the slab row k is added to image row ds_rows[k] after the
    FFN residual. ``rows`` restricts the computation to those output rows
    (K/V are still formed for every row); other rows of the result are zero.
    ``taps`` (a dict) receives the intermediates.
    """
    x = _np(x, dtype)
    S = x.shape[0]
    nh, hd = cfg.n_heads, cfg.head_dim
    angles = mrope_angles(pos, cfg.rope_theta, hd, cfg.mrope_section)
    sel = np.arange(S) if rows is None else np.asarray(rows)
    q, k, v = qkv(cfg, W, x, angles, dtype, None if rows is None else sel)
    o = attention(q, k, v, rows)
    h = np.zeros_like(x)
    h[sel] = o_residual(W, o[sel].reshape(len(sel), nh * hd), x[sel], dtype)
    a = ffn_act(cfg, W, h[sel], dtype)
    out = np.zeros_like(x)
    out[sel] = down_residual(W, a, h[sel], dtype)
    if ds_slab is not None:
        slab = _np(ds_slab, dtype)
        ds_rows = np.asarray(ds_rows)
        if len(ds_rows) == 0 or len(ds_rows) != slab.shape[0]:
            raise OracleError("DeepStack slab rows and image rows disagree")
        if ds_rows.max() >= S or ds_rows.min() < 0:
            raise OracleError("DeepStack image row out of range")
        keep = np.isin(ds_rows, sel)
        out[ds_rows[keep]] += slab[keep]
    if taps is not None:
        taps.update(q=q, k=k, v=v, o=o, h=h, act=a)
    return out


def stack(cfg: Config, layers: List[Dict], x, pos: np.ndarray, ds_slabs=(), ds_rows=None,
          final_norm=None, n_deepstack: int = 3, dtype=np.float64) -> np.ndarray:
    """n layers, DeepStack slab l after layer l, then the optional final RMSNorm.

    With images present the caller supplies at least ``n_deepstack`` slabs
    (hf2q ``forward_text_prefill_logits_last`` validation); without a final
    norm the unnormalised residual stream is returned (the 32B encoder).
    """
    h = _np(x, dtype)
    if len(ds_slabs):
        if len(ds_slabs) < n_deepstack:
            raise OracleError("fewer DeepStack slabs than DeepStack layers")
        if ds_rows is None or len(ds_rows) == 0:
            raise OracleError("DeepStack slabs given without image rows")
    for li, W in enumerate(layers):
        slab = ds_slabs[li] if li < len(ds_slabs) else None
        h = layer(cfg, W, h, pos, slab, ds_rows if slab is not None else None, dtype)
    if final_norm is not None:
        h = rms_norm(h, _np(final_norm, dtype), cfg.rms_eps)
    return h


# ---------------------------------------------------------------------------
# KV cache and incremental decode
# ---------------------------------------------------------------------------
#
# hf2q ``qwen3vl_text/forward.rs``, module doc "Why no KV cache yet": the
# first generation loop re-runs the whole prefill over prompt + tokens
# decoded so far and keeps the last row; a KV cache only saves that work.
# So a decoded token's output is, by definition, the last row of the prefill
# over the extended sequence. The cache form below reaches the same numbers:
# the K/V of the earlier rows do not depend on the new row (the layer is
# causal), so they are computed once and kept.

def text_positions_after(next_pos: int, n: int) -> np.ndarray:
    """Positions of n text tokens that follow a prompt: all three axes equal
    next_pos + i (inferencelayer ``vision.rs``: generation resumes one past
    the largest position any axis reached, and a text token advances every
    axis by one)."""
    p = np.arange(next_pos, next_pos + n, dtype=np.int64)
    return np.stack([p, p, p])


def kv_rows(cfg: Config, W: Dict, x, pos: np.ndarray, dtype=np.float64):
    """What a cache holds for rows 0..S-1 of one layer: K after the per-head
    norm and MRoPE, and V, both [S, nkv, hd] (the k and v of ``qkv``)."""
    x = _np(x, dtype)
    angles = mrope_angles(pos, cfg.rope_theta, cfg.head_dim, cfg.mrope_section)
    _, k, v = qkv(cfg, W, x, angles, dtype, q_rows=np.zeros(0, dtype=np.int64))
    return k, v


def layer_decode(cfg: Config, W: Dict, x_new, pos_new: np.ndarray, k_cache: Sequence,
                 v_cache: Sequence, dtype=np.float64, taps: Optional[Dict] = None):
    """One new token for each of B sequences through one layer.

    x_new [B, H] are the new tokens' layer inputs, pos_new [3, B] their
    positions, and k_cache[b] / v_cache[b] ([L_b, nkv, hd], L_b >= 0) the
    cached K/V of sequence b's earlier rows. The new row attends to every
    cached row and to itself (the causal row of the extended sequence).
    Returns (x' [B, H], k_new [B, nkv, hd], v_new [B, nkv, hd]); k_new and
    v_new are the rows a cache appends.
    """
    x_new = _np(x_new, dtype)
    B = x_new.shape[0]
    nh, nkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    out = np.zeros_like(x_new)
    k_new = np.zeros((B, nkv, hd), dtype=x_new.dtype)
    v_new = np.zeros_like(k_new)
    o_all = np.zeros((B, nh, hd), dtype=x_new.dtype)
    for b in range(B):
        angles = mrope_angles(np.asarray(pos_new)[:, b:b + 1], cfg.rope_theta, hd,
                              cfg.mrope_section)
        q, k, v = qkv(cfg, W, x_new[b:b + 1], angles, dtype)
        kc = _np(k_cache[b], dtype).reshape(-1, nkv, hd)
        vc = _np(v_cache[b], dtype).reshape(-1, nkv, hd)
        L = kc.shape[0]
        K = np.concatenate([kc, k], axis=0)
        V = np.concatenate([vc, v], axis=0)
        Q = np.zeros((L + 1, nh, hd), dtype=q.dtype)
        Q[L] = q[0]
        o = attention(Q, K, V, rows=np.array([L]))[L]
        h = o_residual(W, o.reshape(1, nh * hd), x_new[b:b + 1], dtype)
        a = ffn_act(cfg, W, h, dtype)
        out[b] = down_residual(W, a, h, dtype)[0]
        k_new[b], v_new[b], o_all[b] = k[0], v[0], o
    if taps is not None:
        taps.update(o=o_all, k=k_new, v=v_new)
    return out, k_new, v_new


def stack_prefill_kv(cfg: Config, layers: List[Dict], x, pos: np.ndarray, ds_slabs=(),
                     ds_rows=None, final_norm=None, n_deepstack: int = 3, dtype=np.float64):
    """``stack`` that also returns each layer's cache rows [(k, v), ...]:
    layer l's K/V are formed from layer l's own input."""
    h = _np(x, dtype)
    if len(ds_slabs):
        if len(ds_slabs) < n_deepstack:
            raise OracleError("fewer DeepStack slabs than DeepStack layers")
        if ds_rows is None or len(ds_rows) == 0:
            raise OracleError("DeepStack slabs given without image rows")
    caches = []
    for li, W in enumerate(layers):
        caches.append(kv_rows(cfg, W, h, pos, dtype))
        slab = ds_slabs[li] if li < len(ds_slabs) else None
        h = layer(cfg, W, h, pos, slab, ds_rows if slab is not None else None, dtype)
    if final_norm is not None:
        h = rms_norm(h, _np(final_norm, dtype), cfg.rms_eps)
    return h, caches


def stack_decode(cfg: Config, layers: List[Dict], x_new, pos_new: np.ndarray,
                 caches: Sequence, final_norm=None, dtype=np.float64):
    """One new token per sequence through every layer, then the optional final
    norm. caches[l] = (k_cache, v_cache), each a per-sequence list as in
    ``layer_decode``. Returns (y [B, H], [(k_new, v_new) per layer])."""
    h = _np(x_new, dtype)
    new = []
    for li, W in enumerate(layers):
        kc, vc = caches[li]
        h, kn, vn = layer_decode(cfg, W, h, pos_new, kc, vc, dtype)
        new.append((kn, vn))
    if final_norm is not None:
        h = rms_norm(h, _np(final_norm, dtype), cfg.rms_eps)
    return h, new


# ---------------------------------------------------------------------------
# The steps either side of the layers: embedding gather with the soft-token
# splice, and the final norm + LM head
# ---------------------------------------------------------------------------

def embed(table, tokens: Sequence[int], soft_rows: Sequence[int] = (), soft=None,
          dtype=np.float64) -> np.ndarray:
    """x[p] = table[tokens[p]], then x[soft_rows[k]] = soft[k] (the spliced rows).

    hf2q ``qwen3vl_text/forward.rs``, ``forward_text_prefill_logits_last``,
    step 1: the token embedding lookup, then every soft-token injection
    overwrites its rows with the supplied embeddings. The injections must lie
    inside the prompt and must not overlap; here they are given as one list of
    destination rows with one embedding row each (a range [s, e) is the rows
    s..e-1), so "overlap" is a repeated row. A token id outside the table is
    an error as well.
    """
    table = _np(table, dtype)
    tokens = np.asarray(tokens, dtype=np.int64)
    S, vocab = len(tokens), table.shape[0]
    if S == 0:
        raise OracleError("empty token list")
    if tokens.min() < 0 or tokens.max() >= vocab:
        raise OracleError("token id outside the embedding table")
    x = table[tokens].copy()
    soft_rows = np.asarray(soft_rows, dtype=np.int64)
    if len(soft_rows):
        soft = _np(soft, dtype)
        if soft.shape[0] != len(soft_rows):
            raise OracleError("soft-token rows and embeddings disagree")
        if soft_rows.min() < 0 or soft_rows.max() >= S:
            raise OracleError("soft-token row outside the prompt")
        if len(np.unique(soft_rows)) != len(soft_rows):
            raise OracleError("soft-token rows overlap")
        x[soft_rows] = soft
    return x


def lm_head(cfg: Config, x_rows, final_norm, weight, dtype=np.float64) -> np.ndarray:
    """logits = RMSNorm(x, final_norm) W^T for each given row ([rows, vocab]).

    hf2q ``qwen3vl_text/forward.rs``, step 4: the last position's residual
    row goes through the final RMSNorm and the LM head; W is the output
    weight, or the token embedding table itself when the embeddings are tied.
    """
    xn = rms_norm(_np(x_rows, dtype), _np(final_norm, dtype), cfg.rms_eps)
    return xn @ _np(weight, dtype).T
