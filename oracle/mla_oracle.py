"""fp64 CPU oracle for MLA decode: the plain, non-absorbed definition.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only the tests, the package entry's smoke check and the benchmark's
CPU-baseline leg use it.  It shares no code with the CUDA path.

What it computes, and where each step is stated:

* Per-head key/value reconstruction from the cached latent, K = c W_K^(h)
  and V = c W_V^(h) -- "Understanding MLA (Multi-head Latent Attention)",
  section 2 (the formal definition) and Phase B, step B1.
* Rotary embedding of the 64-wide rope key, shared by all heads (Phase B,
  step B2) and of the query's rope half at the query's own position
  (Phase C, step C2).  The pair layout and base are not fixed by the pages;
  this oracle takes interleaved pairs (x[2i], x[2i+1]) rotated by
  pos * base^(-2i/d_R), base 10000 (a reading: the pages leave it open).
* Concatenation Q = [Q_nope || Q_rope], K = [K_nope || K_rope] and
  softmax(Q K^T / sqrt(qk_nope + d_R)) V (Phase D, steps D1-D2;
  "Multi-Head Latent Attention", section 3, the sketch's last two lines).
  decode_* stop at the per-head value vector; output_projection concatenates
  the heads and projects to the hidden width ("Understanding MLA", Phase D
  step D2).
* The append step: one projection x W_DKV to d_c + d_R values, split into
  the latent and the rope key, rope key rotated at the token's position
  (Phase A, step A1; "Multi-head latent attention" on aicassindra,
  "End-to-end flow"); optionally the latent alone RMS-normalised first
  (Phase A, step A2; epsilon 1e-6, which the pages do not give).
* Decode over a selected subset of each query's cached keys (the top-k
  selection of "Multi-Head Latent Attention", section 4; the selector itself
  is not part of this oracle).
* An absorbed variant, used only to check the regrouping
  Q_nope . (W_K c) = (Q_nope W_K) . c ("Understanding MLA", section 4).

Causality: query j of a sequence holding ``L`` cached keys (its own entry
included) sits at position p = L - n_q + j and attends keys 0..p.

Every array is converted to float64 on entry; numpy matmul is the only
library primitive used for contractions.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):                   # torch tensor (any dtype)
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# RoPE ("Understanding MLA", Phase B step B2 and Phase C step C2)
# ---------------------------------------------------------------------------
def rope_frequencies(d_rope: int, base: float = 10000.0) -> np.ndarray:
    """theta_i = base^(-2i/d_R) for pair i = 0 .. d_R/2 - 1."""
    i = np.arange(d_rope // 2, dtype=np.float64)
    return base ** (-2.0 * i / d_rope)


def rope(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate each interleaved pair (x[2i], x[2i+1]) by angle pos * theta_i.

    ``x`` has shape [..., d_R]; ``pos`` broadcasts against ``x[..., 0]``.
    """
    x = _f64(x)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_frequencies(d, base)
    cos, sin = np.cos(ang), np.sin(ang)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), dtype=np.float64)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


def rope_cache(k_rope_raw, lens, base: float = 10000.0) -> np.ndarray:
    """Rotate cache slot n of every sequence at position n (slots >= len kept)."""
    k = _f64(k_rope_raw).copy()
    for b, L in enumerate(np.asarray(lens).tolist()):
        k[b, :L] = rope(k[b, :L], np.arange(L), base)
    return k


# ---------------------------------------------------------------------------
# Decode, naive (materialised) form
# ---------------------------------------------------------------------------
def softmax(s: np.ndarray) -> np.ndarray:
    """Numerically stable softmax of a 1-D score vector."""
    e = np.exp(s - np.max(s))
    return e / np.sum(e)


def decode_naive(q_nope, q_rope, W_uk, W_uv, c_kv, k_rope_rot, lens, n_q: int,
                 scale: float, base: float = 10000.0, *, batches=None, heads=None,
                 pos_offset: int = 0, return_weights: bool = False):
    """Naive MLA decode.

    q_nope [B][n_q][H][qk_nope], q_rope [B][n_q][H][d_R] (not rotated),
    W_uk [H][d_c][qk_nope], W_uv [H][d_c][v_dim], c_kv [B][cap][d_c],
    k_rope_rot [B][cap][d_R] (already rotated at its slot position, as the
    cache stores it), lens [B].  Returns out [B][n_q][H][v_dim] (float64) for
    the selected batches/heads (others stay zero).  ``pos_offset`` shifts every
    position -- keys and queries -- by the same amount; the cache's rope keys
    are then re-rotated by that offset, which is what a cache built at shifted
    positions would hold.
    """
    q_nope, q_rope = _f64(q_nope), _f64(q_rope)
    W_uk, W_uv = _f64(W_uk), _f64(W_uv)
    lens = [int(v) for v in np.asarray(lens).tolist()]
    B, _, H, _ = q_nope.shape
    v_dim = W_uv.shape[-1]
    batches = range(B) if batches is None else batches
    heads = range(H) if heads is None else heads
    out = np.zeros((B, n_q, H, v_dim), dtype=np.float64)
    weights = {}
    for b in batches:
        L = lens[b]
        c = _f64(c_kv[b, :L])                                   # [L][d_c]
        k_r = _f64(k_rope_rot[b, :L])                           # [L][d_R]
        if pos_offset:
            k_r = rope(k_r, np.full(L, pos_offset), base)
        for h in heads:
            K_nope = c @ W_uk[h]                                # [L][qk_nope]
            V = c @ W_uv[h]                                     # [L][v_dim]
            for j in range(n_q):
                p = L - n_q + j                                 # query position
                q = np.concatenate([q_nope[b, j, h],
                                    rope(q_rope[b, j, h], p + pos_offset, base)])
                K = np.concatenate([K_nope[: p + 1], k_r[: p + 1]], axis=1)
                s = (K @ q) * scale
                w = softmax(s)
                out[b, j, h] = w @ V[: p + 1]
                if return_weights:
                    weights[(b, j, h)] = w
    if return_weights:
        return out, weights
    return out


def decode_sparse(q_nope, q_rope, W_uk, W_uv, c_kv, k_rope_rot, lens, sel, n_sel, n_q: int,
                  scale: float, base: float = 10000.0, *, batches=None, heads=None):
    """Decode restricted to a selected subset of each query's cached keys.

    "Multi-Head Latent Attention", section 4: a selector picks a top-k subset
    of the cached latents per query and MLA runs unchanged on that subset.
    sel [B][n_q][max_sel] holds distinct cache slots (each <= the query's
    position p), n_sel [B][n_q] how many leading entries are used.  Per head:
    the same naive K = c W_K, V = c W_V, RoPE and softmax as decode_naive, over
    the selected rows only, in the order given.
    """
    q_nope, q_rope = _f64(q_nope), _f64(q_rope)
    W_uk, W_uv = _f64(W_uk), _f64(W_uv)
    lens = [int(v) for v in np.asarray(lens).tolist()]
    sel, n_sel = np.asarray(sel), np.asarray(n_sel)
    B, _, H, _ = q_nope.shape
    batches = range(B) if batches is None else batches
    heads = range(H) if heads is None else heads
    out = np.zeros((B, n_q, H, W_uv.shape[-1]), dtype=np.float64)
    for b in batches:
        L = lens[b]
        for j in range(n_q):
            p = L - n_q + j
            rows = sel[b, j, : int(n_sel[b, j])]
            c = _f64(c_kv[b, rows])                             # [k][d_c]
            k_r = _f64(k_rope_rot[b, rows])                     # [k][d_R]
            for h in heads:
                q = np.concatenate([q_nope[b, j, h], rope(q_rope[b, j, h], p, base)])
                K = np.concatenate([c @ W_uk[h], k_r], axis=1)
                w = softmax((K @ q) * scale)
                out[b, j, h] = w @ (c @ W_uv[h])
    return out


def absorbed_query(q_nope, q_rope, W_uk_h, p, base: float = 10000.0) -> np.ndarray:
    """q_lat = [W_K^(h) q_nope || RoPE(q_rope, p)]: the key up-projection moved to
    the query side ("Understanding MLA", section 4)."""
    return np.concatenate([_f64(W_uk_h) @ _f64(q_nope), rope(q_rope, p, base)])


def latent_attention(q_lat, c, k_rope_rot, scale: float):
    """Softmax-weighted latent for one query against visible cache rows:
    returns (o_lat, lse) with lse = log sum_n exp(s_n) (natural log)."""
    s = (np.concatenate([_f64(c), _f64(k_rope_rot)], axis=1) @ q_lat) * scale
    w = softmax(s)
    mx = np.max(s)
    return w @ _f64(c), mx + np.log(np.sum(np.exp(s - mx)))


def decode_absorbed(q_nope, q_rope, W_uk, W_uv, c_kv, k_rope_rot, lens, n_q: int,
                    scale: float, base: float = 10000.0, *, batches=None, heads=None,
                    return_intermediates: bool = False):
    """Absorbed form: score against the latent directly, up-project after.

    The value up-projection is applied to the softmax-weighted latent
    ("Multi-head latent attention", aicassindra, "End-to-end flow").  Used to
    check the algebra and to give the intermediate results of the absorbed
    path (absorbed queries, latent outputs).
    """
    q_nope, q_rope = _f64(q_nope), _f64(q_rope)
    W_uk, W_uv = _f64(W_uk), _f64(W_uv)
    lens = [int(v) for v in np.asarray(lens).tolist()]
    B, _, H, _ = q_nope.shape
    batches = range(B) if batches is None else batches
    heads = range(H) if heads is None else heads
    out = np.zeros((B, n_q, H, W_uv.shape[-1]), dtype=np.float64)
    inter = {}
    for b in batches:
        L = lens[b]
        c = _f64(c_kv[b, :L])
        k_r = _f64(k_rope_rot[b, :L])
        for h in heads:
            for j in range(n_q):
                p = L - n_q + j
                q_lat = absorbed_query(q_nope[b, j, h], q_rope[b, j, h], W_uk[h], p, base)
                o_lat, lse = latent_attention(q_lat, c[: p + 1], k_r[: p + 1], scale)
                out[b, j, h] = o_lat @ W_uv[h]
                if return_intermediates:
                    inter[(b, j, h)] = (q_lat, o_lat, lse)
    if return_intermediates:
        return out, inter
    return out


# ---------------------------------------------------------------------------
# Output projection ("Understanding MLA", Phase D step D2)
# ---------------------------------------------------------------------------
def output_projection(out, W_O) -> np.ndarray:
    """The per-head outputs concatenated head after head and projected to the
    hidden width: y[t] = [out[t][0] || out[t][1] || ...] W_O.

    out [T][H][v_dim], W_O [H * v_dim][hidden]; returns y [T][hidden].
    """
    out = _f64(out)
    T, H, v = out.shape
    return out.reshape(T, H * v) @ _f64(W_O)


# ---------------------------------------------------------------------------
# Append ("Understanding MLA", Phase A step A1, Phase B step B2)
# ---------------------------------------------------------------------------
RMS_EPS = 1e-6   # not given by the pages: the usual RMSNorm epsilon (a reading)


def rms_norm(c, gamma, eps: float = RMS_EPS) -> np.ndarray:
    """RMSNorm of each row: gamma * c / sqrt(mean(c^2) + eps), one shared RMS
    over the whole row ("Understanding MLA", Phase A step A2)."""
    c = _f64(c)
    rms = np.sqrt(np.mean(c * c, axis=-1, keepdims=True) + eps)
    return _f64(gamma) * c / rms


def append_rows(x, W_dkv, positions, d_c: int, base: float = 10000.0, rms_gamma=None,
                eps: float = RMS_EPS) -> np.ndarray:
    """Cache rows for new tokens: [latent (d_c) || rotated rope key (d_R)].

    x [M][hidden], W_dkv [hidden][d_c + d_R], positions [M].  One projection
    to d_c + d_R values, split into the latent (first d_c) and the rope key
    (last d_R); only the rope key is rotated, at the token's position.  With
    ``rms_gamma`` [d_c] the latent alone is RMS-normalised before it is cached
    and the rope key is left as it is ("Understanding MLA", Phase A step A2).
    """
    y = _f64(x) @ _f64(W_dkv)                                   # [M][d_c + d_R]
    rows = y.copy()
    if rms_gamma is not None:
        rows[:, :d_c] = rms_norm(y[:, :d_c], rms_gamma, eps)
    rows[:, d_c:] = rope(y[:, d_c:], np.asarray(positions), base)
    return rows


def cache_after_append(c_kv, k_rope_rot, rows, positions, n_new: int, d_c: int):
    """Write appended rows into (fp64 copies of) the cache at their slots."""
    c = _f64(c_kv).copy()
    k = _f64(k_rope_rot).copy()
    pos = np.asarray(positions).reshape(-1, n_new)
    for b in range(pos.shape[0]):
        for i in range(n_new):
            r = rows[b * n_new + i]
            c[b, pos[b, i]] = r[:d_c]
            k[b, pos[b, i]] = r[d_c:]
    return c, k


def decode_step(inp: dict, n_q: int, d_c: int, scale: float, base: float = 10000.0,
                *, batches=None, heads=None) -> np.ndarray:
    """Whole decode step on generated inputs: (append,) then attend.

    ``inp`` holds the stored inputs (see the input generator): the cache's
    rope keys are raw and are rotated at their slot positions first; with an
    ``x`` entry the new tokens are appended before attention ("Multi-head
    latent attention", aicassindra, "End-to-end flow": append, then attend).
    """
    lens = inp["seq_lens"]
    if "x" in inp:
        old = np.asarray(inp["old_lens"])
        k_rot = rope_cache(inp["k_rope"], old, base)
        rows = append_rows(inp["x"], inp["W_dkv"], inp["positions"], d_c, base)
        n_new = rows.shape[0] // len(old)
        c, k_rot = cache_after_append(inp["c_kv"], k_rot, rows, inp["positions"], n_new, d_c)
    else:
        k_rot = rope_cache(inp["k_rope"], lens, base)
        c = inp["c_kv"]
    return decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], c, k_rot,
                        lens, n_q, scale, base, batches=batches, heads=heads)


# ---------------------------------------------------------------------------
# Storage arithmetic ("Understanding MLA", section 5; akshathtiwari, MLA blog)
# ---------------------------------------------------------------------------
def cache_values_per_token(d_c: int, d_rope: int) -> int:
    """Values one token caches per layer: the latent plus the rope key."""
    return d_c + d_rope


def mha_values_per_token(heads: int, qk_dim: int, v_dim: int) -> int:
    """Values a per-head full key/value cache would hold per token per layer."""
    return heads * (qk_dim + v_dim)
