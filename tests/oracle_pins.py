"""Pins for the fp64 oracle: facts fixed by the pages or by mathematics.

Each ``pin_*`` takes the oracle module and raises AssertionError when the
oracle disagrees.  None of them re-types the oracle's own formula: they use
closed forms, invariants, a different formulation (complex multiplication
for RoPE, torch's scaled-dot-product attention for the whole attention),
brute force on tiny inputs, or numbers printed on the pages.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import scipy.special
import torch

from mla_latent_kv_43_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _close(a, b, rtol=1e-12, atol=1e-12):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    ref = max(np.max(np.abs(b)) if b.size else 0.0, 1e-300)
    assert err <= atol + rtol * ref, f"max|d|={err:.3e} max|ref|={ref:.3e}"


def _np(t):
    return t.double().numpy()


# --------------------------------------------------------------------- RoPE
def pin_rope_identity_at_zero(O):
    """Rotation by angle 0 is the identity (position 0)."""
    x = np.random.default_rng(1).standard_normal((5, 16))
    _close(O.rope(x, 0), x, rtol=0, atol=0)


def pin_rope_preserves_norm(O):
    """A rotation preserves every pair's length, hence the vector's norm."""
    x = np.random.default_rng(2).standard_normal((7, 64))
    y = O.rope(x, np.arange(7) * 1000 + 3)
    _close(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-14)


def pin_rope_2d_is_plane_rotation(O):
    """With d_R = 2, theta_0 = 1: the textbook 2-D rotation by pos radians."""
    x = np.array([0.3, -1.7])
    for p in (0, 1, 2, 5, 100, 131071):
        R = np.array([[math.cos(p), -math.sin(p)], [math.sin(p), math.cos(p)]])
        _close(O.rope(x, p), R @ x, rtol=1e-14, atol=1e-15)


def pin_rope_complex_form(O):
    """Interleaved pair i as the complex number x[2i] + i x[2i+1], multiplied by
    exp(i * pos * base^(-2i/d)): the same map written another way."""
    rng = np.random.default_rng(3)
    for d in (4, 16, 64):
        x = rng.standard_normal((6, d))
        pos = np.array([0, 1, 7, 4095, 4096, 131071])
        z = x[:, 0::2] + 1j * x[:, 1::2]
        freq = np.power(10000.0, -np.arange(0, d, 2) / d)
        zr = z * np.exp(1j * pos[:, None] * freq[None, :])
        ref = np.empty_like(x)
        ref[:, 0::2], ref[:, 1::2] = zr.real, zr.imag
        _close(O.rope(x, pos), ref, rtol=1e-12, atol=1e-12)


def pin_rope_relative(O):
    """(R_m q) . (R_n k) = q^T R_(n-m) k: the score sees only the offset
    ("Understanding MLA", section 4)."""
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in ((0, 0), (3, 10), (4097, 12), (100000, 99999)):
        lhs = O.rope(q, m) @ O.rope(k, n)
        rhs = q @ O.rope(k, n - m)
        _close(lhs, rhs, rtol=1e-10, atol=1e-10)


# ------------------------------------------------------------ decode checks
def _tiny_inputs(seed=0, n_q=1, lens=(5, 9), qk_nope=6, v_dim=5, heads=3, d_c=8, d_rope=4):
    w = gen.tiny("fp32", lens=lens, n_q=n_q, seed=seed, qk_nope=qk_nope, v_dim=v_dim,
                 heads=heads, d_c=d_c, d_rope=d_rope)
    return w, gen.generate(w)


def _rot_cache(O, inp, lens=None):
    return O.rope_cache(inp["k_rope"], inp["seq_lens"] if lens is None else lens)


def pin_absorbed_equals_naive(O):
    """Moving W_K to the query side is an exact regrouping ("Understanding MLA",
    section 4): absorbed and materialised decode agree to rounding."""
    for n_q in (1, 2):
        w, inp = _tiny_inputs(seed=5, n_q=n_q, lens=(3, 11))
        k = _rot_cache(O, inp)
        a = O.decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"],
                           k, inp["seq_lens"], n_q, w.softmax_scale)
        b = O.decode_absorbed(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"],
                              inp["c_kv"], k, inp["seq_lens"], n_q, w.softmax_scale)
        _close(a, b, rtol=1e-12)


def pin_length_one_returns_value(O):
    """One visible key: softmax weight 1, output = c_0 W_V^(h) for any query."""
    w, inp = _tiny_inputs(seed=6, lens=(1, 1))
    out = O.decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"],
                         _rot_cache(O, inp), inp["seq_lens"], 1, w.softmax_scale)
    c, Wv = _np(inp["c_kv"]), _np(inp["W_uv"])
    for b in range(2):
        for h in range(w.heads):
            ref = [sum(c[b, 0, i] * Wv[h, i, v] for i in range(w.d_c)) for v in range(w.v_dim)]
            _close(out[b, 0, h], ref, rtol=1e-14)


def pin_zero_query_is_uniform_mean(O):
    """q = 0: all scores 0, uniform weights, output = mean(c_0..c_p) W_V^(h)."""
    w, inp = _tiny_inputs(seed=7, lens=(4, 9), n_q=2)
    inp["q_nope"].zero_()
    inp["q_rope"].zero_()
    out = O.decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"],
                         _rot_cache(O, inp), inp["seq_lens"], 2, w.softmax_scale)
    c, Wv = _np(inp["c_kv"]), _np(inp["W_uv"])
    for b, L in enumerate((4, 9)):
        for j in range(2):
            p = L - 2 + j
            for h in range(w.heads):
                _close(out[b, j, h], c[b, : p + 1].mean(axis=0) @ Wv[h], rtol=1e-13)


def pin_weights_sum_to_one(O):
    w, inp = _tiny_inputs(seed=8, lens=(6, 13), n_q=2)
    _, ws = O.decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"],
                           _rot_cache(O, inp), inp["seq_lens"], 2, w.softmax_scale,
                           return_weights=True)
    for (b, j, h), wt in ws.items():
        L = (6, 13)[b]
        assert wt.shape == (L - 2 + j + 1,), (wt.shape, b, j)
        assert np.all(wt >= 0)
        assert abs(wt.sum() - 1.0) < 1e-14


def pin_global_shift_invariance(O):
    """Shifting every position by the same amount leaves the output unchanged
    (RoPE scores depend on n - m only)."""
    w, inp = _tiny_inputs(seed=9, lens=(7, 12), n_q=2)
    k = _rot_cache(O, inp)
    args = (inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"], k,
            inp["seq_lens"], 2, w.softmax_scale)
    _close(O.decode_naive(*args), O.decode_naive(*args, pos_offset=777), rtol=1e-10)


def pin_causal(O):
    """Query j sees keys 0..L-n_q+j: changing the last entry changes only the
    last query's output."""
    w, inp = _tiny_inputs(seed=10, lens=(6, 9), n_q=2)
    k = _rot_cache(O, inp)
    base = O.decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"],
                          k, inp["seq_lens"], 2, w.softmax_scale)
    c2 = inp["c_kv"].clone()
    k2 = k.copy()
    for b, L in enumerate((6, 9)):
        c2[b, L - 1] += 3.0
        k2[b, L - 1] += 2.0
    mod = O.decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], c2, k2,
                         inp["seq_lens"], 2, w.softmax_scale)
    _close(mod[:, 0], base[:, 0], rtol=0, atol=0)
    assert np.max(np.abs(mod[:, 1] - base[:, 1])) > 1e-3


def pin_rope_only_scores_match_scipy_softmax(O):
    """W_K = 0 leaves only the rope dot in the score; the weights are then
    scipy's softmax of scale * (R_n k_n) . (R_p q_rope).  The rope key is
    never up-projected ("Understanding MLA", section 7)."""
    w, inp = _tiny_inputs(seed=11, lens=(8, 3))
    inp["W_uk"].zero_()
    k = _rot_cache(O, inp)
    out = O.decode_naive(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"],
                         k, inp["seq_lens"], 1, w.softmax_scale)
    c, Wv, qr, kraw = _np(inp["c_kv"]), _np(inp["W_uv"]), _np(inp["q_rope"]), _np(inp["k_rope"])
    for b, L in enumerate((8, 3)):
        p = L - 1
        kz = kraw[b, :L, 0::2] + 1j * kraw[b, :L, 1::2]
        freq = np.power(10000.0, -np.arange(0, w.d_rope, 2) / w.d_rope)
        kz = kz * np.exp(1j * np.arange(L)[:, None] * freq)
        for h in range(w.heads):
            qz = (qr[b, 0, h, 0::2] + 1j * qr[b, 0, h, 1::2]) * np.exp(1j * p * freq)
            s = (kz.real @ qz.real + kz.imag @ qz.imag) * w.softmax_scale
            ref = scipy.special.softmax(s) @ (c[b, :L] @ Wv[h])
            _close(out[b, 0, h], ref, rtol=1e-12)


def _torch_rope(x, pos, base=10000.0):
    """RoPE through torch complex arithmetic (independent of the oracle)."""
    d = x.shape[-1]
    z = torch.view_as_complex(x.reshape(*x.shape[:-1], d // 2, 2).contiguous())
    freq = base ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
    ang = pos.to(torch.float64)[..., None] * freq
    return torch.view_as_real(z * torch.polar(torch.ones_like(ang), ang)).reshape(x.shape)


def _torch_reference(w, inp):
    """Whole decode step written with torch float64 ops and SDPA."""
    f = lambda k: inp[k].to(torch.float64)
    c, kr = f("c_kv").clone(), f("k_rope").clone()
    lens = inp["seq_lens"].long()
    B = w.batch
    slots = torch.arange(w.capacity)
    kr = _torch_rope(kr, slots.expand(B, -1))
    if w.n_new:
        y = f("x") @ f("W_dkv")
        pos = inp["positions"].long()
        y_r = _torch_rope(y[:, w.d_c:], pos)
        for r in range(B * w.n_new):
            b = r // w.n_new
            c[b, pos[r]] = y[r, : w.d_c]
            kr[b, pos[r]] = y_r[r]
    out = torch.zeros(B, w.n_q, w.heads, w.v_dim, dtype=torch.float64)
    for b in range(B):
        L = int(lens[b])
        Kn = torch.einsum("ld,hdk->hlk", c[b, :L], f("W_uk"))
        V = torch.einsum("ld,hdv->hlv", c[b, :L], f("W_uv"))
        K = torch.cat([Kn, kr[b, :L].expand(w.heads, L, w.d_rope)], dim=-1)
        qpos = torch.arange(L - w.n_q, L)
        qr = _torch_rope(f("q_rope")[b].transpose(0, 1), qpos.expand(w.heads, -1))
        Q = torch.cat([f("q_nope")[b].transpose(0, 1), qr], dim=-1)        # [H][n_q][192]
        mask = slots[:L][None, :] <= qpos[:, None]                          # [n_q][L]
        o = torch.nn.functional.scaled_dot_product_attention(
            Q, K, V, attn_mask=mask, scale=w.softmax_scale)
        out[b] = o.transpose(0, 1)
    return out.numpy()


def pin_whole_step_matches_torch_sdpa(O):
    """The whole step from raw stored inputs (rope keys rotated at their slot,
    queries at L - n_q + j, causal mask) against torch's SDPA in float64."""
    for n_q, lens in ((1, (5, 9)), (2, (4, 11)), (3, (3, 6))):
        w, inp = _tiny_inputs(seed=12 + n_q, lens=lens, n_q=n_q)
        got = O.decode_step(inp, n_q, w.d_c, w.softmax_scale)
        _close(got, _torch_reference(w, inp), rtol=1e-11)


def pin_step_with_append_matches_torch(O):
    """Append-then-attend: new rows from x W_DKV, split, rope key rotated at the
    new positions, then two causal queries (the second sees the first)."""
    w = gen.tiny("fp32", lens=(6, 9), capacity=10, n_q=2, n_new=2, hidden=12, seed=21)
    inp = gen.generate(w)
    got = O.decode_step(inp, 2, w.d_c, w.softmax_scale)
    _close(got, _torch_reference(w, inp), rtol=1e-11)


def pin_append_brute_force(O):
    """Append rows by explicit loops on a tiny input: latent = first d_c
    outputs of the one projection, rope key = the last d_R, rotated."""
    rng = np.random.default_rng(13)
    M, hidden, d_c, d_r = 3, 5, 4, 4
    x = rng.standard_normal((M, hidden))
    W = rng.standard_normal((hidden, d_c + d_r))
    pos = np.array([0, 5, 4097])
    rows = O.append_rows(x, W, pos, d_c)
    for m in range(M):
        y = [sum(x[m, k] * W[k, n] for k in range(hidden)) for n in range(d_c + d_r)]
        _close(rows[m, :d_c], y[:d_c], rtol=1e-13)
        for i in range(d_r // 2):
            ang = pos[m] * 10000.0 ** (-2 * i / d_r)
            a, b = y[d_c + 2 * i], y[d_c + 2 * i + 1]
            _close(rows[m, d_c + 2 * i], a * math.cos(ang) - b * math.sin(ang), rtol=1e-12, atol=1e-13)
            _close(rows[m, d_c + 2 * i + 1], a * math.sin(ang) + b * math.cos(ang), rtol=1e-12, atol=1e-13)


def pin_append_rms_norm(O):
    """RMSNorm of the latent at append ("Understanding MLA", Phase A step A2):
    with gamma = 1 the cached latent has root-mean-square 1 (up to eps), it is
    unchanged when x is scaled (the norm divides the scale out), gamma scales it
    linearly, the rope key is exactly the un-normalised one, and explicit loops
    on a tiny input give the same values."""
    rng = np.random.default_rng(31)
    M, hidden, d_c, d_r = 4, 7, 6, 4
    x = rng.standard_normal((M, hidden))
    W = rng.standard_normal((hidden, d_c + d_r))
    pos = np.array([0, 3, 17, 4096])
    ones = np.ones(d_c)
    rows = O.append_rows(x, W, pos, d_c, rms_gamma=ones, eps=0.0)
    _close(np.sqrt(np.mean(rows[:, :d_c] ** 2, axis=1)), np.ones(M), rtol=1e-13)
    _close(O.append_rows(7.5 * x, W, pos, d_c, rms_gamma=ones, eps=0.0)[:, :d_c], rows[:, :d_c], rtol=1e-13)
    g = rng.uniform(0.5, 2.0, d_c)
    _close(O.append_rows(x, W, pos, d_c, rms_gamma=g, eps=0.0)[:, :d_c], rows[:, :d_c] * g, rtol=1e-13)
    plain = O.append_rows(x, W, pos, d_c)
    assert np.array_equal(rows[:, d_c:], plain[:, d_c:])
    eps = 1e-6
    rows = O.append_rows(x, W, pos, d_c, rms_gamma=g, eps=eps)
    for m in range(M):
        y = [sum(x[m, k] * W[k, n] for k in range(hidden)) for n in range(d_c)]
        ms = sum(v * v for v in y) / d_c
        _close(rows[m, :d_c], [g[n] * y[n] / math.sqrt(ms + eps) for n in range(d_c)], rtol=1e-13)


def pin_rms_norm_does_not_commute_with_up_projection(O):
    """The page's remark that W RMSNorm(c) != RMSNorm(W c): the norm has to be
    applied to the cached latent itself, before any head's up-projection."""
    rng = np.random.default_rng(32)
    c = rng.standard_normal((3, 8))
    W = rng.standard_normal((8, 5))
    a = O.rms_norm(c, np.ones(8)) @ W
    b = O.rms_norm(c @ W, np.ones(5))
    assert np.max(np.abs(a - b)) > 1e-3


def pin_sparse_decode(O):
    """Decode over selected keys: selecting every visible key gives the dense
    decode, the order of the selected keys does not matter, a single selected
    key returns its value c_k W_V exactly, and explicit loops over a tiny
    selection agree."""
    n_q, lens = 2, (9, 13)
    w, inp = _tiny_inputs(seed=41, lens=lens, n_q=n_q)
    k_rot = O.rope_cache(inp["k_rope"], inp["seq_lens"])
    args = (inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"], k_rot, inp["seq_lens"])
    B, kmax = len(lens), max(lens)
    sel = np.zeros((B, n_q, kmax), dtype=np.int64)
    n_sel = np.zeros((B, n_q), dtype=np.int64)
    for b, L in enumerate(lens):
        for j in range(n_q):
            p = L - n_q + j
            sel[b, j, : p + 1] = np.arange(p + 1)
            n_sel[b, j] = p + 1
    dense = O.decode_naive(*args, n_q, w.softmax_scale)
    _close(O.decode_sparse(*args, sel, n_sel, n_q, w.softmax_scale), dense, rtol=1e-12)
    rng = np.random.default_rng(42)
    shuffled = sel.copy()
    for b in range(B):
        for j in range(n_q):
            shuffled[b, j, : n_sel[b, j]] = rng.permutation(sel[b, j, : n_sel[b, j]])
    _close(O.decode_sparse(*args, shuffled, n_sel, n_q, w.softmax_scale), dense, rtol=1e-12)
    one = np.zeros_like(sel)
    one[:, :, 0] = 2
    got = O.decode_sparse(*args, one, np.ones_like(n_sel), n_q, w.softmax_scale)
    c, W_uv = np.asarray(inp["c_kv"], np.float64), np.asarray(inp["W_uv"], np.float64)
    for b in range(B):
        for h in range(w.heads):
            assert np.array_equal(got[b, :, h], np.stack([c[b, 2] @ W_uv[h]] * n_q))
    # explicit loops: sequence 1, query 1 (position 12), keys {12, 3, 7}
    sub = np.zeros_like(sel)
    sub[1, 1, :3] = [12, 3, 7]
    ns = np.zeros_like(n_sel)
    ns[:, :] = 1
    ns[1, 1] = 3
    got = O.decode_sparse(*args, sub, ns, n_q, w.softmax_scale)
    W_uk = np.asarray(inp["W_uk"], np.float64)
    qn, qr = np.asarray(inp["q_nope"], np.float64), np.asarray(inp["q_rope"], np.float64)
    for h in range(w.heads):
        qrot = [0.0] * w.d_rope
        for i in range(w.d_rope // 2):
            ang = 12 * 10000.0 ** (-2 * i / w.d_rope)
            a, bb = qr[1, 1, h, 2 * i], qr[1, 1, h, 2 * i + 1]
            qrot[2 * i], qrot[2 * i + 1] = a * math.cos(ang) - bb * math.sin(ang), a * math.sin(ang) + bb * math.cos(ang)
        scores = []
        for n in (12, 3, 7):
            kn = [sum(c[1, n, i] * W_uk[h][i][t] for i in range(w.d_c)) for t in range(w.qk_nope)]
            s_ = sum(qn[1, 1, h, t] * kn[t] for t in range(w.qk_nope)) + sum(qrot[t] * k_rot[1, n, t] for t in range(w.d_rope))
            scores.append(s_ * w.softmax_scale)
        mx = max(scores)
        e = [math.exp(v - mx) for v in scores]
        wts = [v / sum(e) for v in e]
        ref = [sum(wts[k] * sum(c[1, n, i] * W_uv[h][i][v] for i in range(w.d_c)) for k, n in enumerate((12, 3, 7)))
               for v in range(w.v_dim)]
        _close(got[1, 1, h], ref, rtol=1e-11)


def pin_output_projection(O):
    """Heads concatenated head-major then projected: the same as summing each
    head's block product, as torch's float64 linear map of the flattened
    heads, and as the absorbed form sum_h o_lat[h] (W_V[h] W_O[h-block]) (the
    value up-projection folded into the output projection, aicassindra
    "Multi-head latent attention", "End-to-end flow")."""
    rng = np.random.default_rng(51)
    T, H, v, hidden = 3, 4, 5, 7
    out = rng.standard_normal((T, H, v))
    W_O = rng.standard_normal((H * v, hidden))
    y = O.output_projection(out, W_O)
    _close(y, sum(out[:, h] @ W_O[h * v:(h + 1) * v] for h in range(H)), rtol=1e-12)
    ref = torch.nn.functional.linear(torch.from_numpy(out.reshape(T, H * v)), torch.from_numpy(W_O.T.copy()))
    _close(y, ref.numpy(), rtol=1e-12)
    # absorbed: through the decode's latent outputs
    w, inp = _tiny_inputs(seed=52, lens=(6, 9), v_dim=v, heads=H)
    k_rot = O.rope_cache(inp["k_rope"], inp["seq_lens"])
    W_O = rng.standard_normal((H * v, hidden))
    outs, inter = O.decode_absorbed(inp["q_nope"], inp["q_rope"], inp["W_uk"], inp["W_uv"], inp["c_kv"], k_rot,
                                    inp["seq_lens"], 1, w.softmax_scale, return_intermediates=True)
    W_uv = np.asarray(inp["W_uv"], np.float64)
    for b in range(2):
        y_b = O.output_projection(outs[b], W_O)[0]
        folded = sum(inter[(b, 0, h)][1] @ (W_uv[h] @ W_O[h * v:(h + 1) * v]) for h in range(H))
        _close(y_b, folded, rtol=1e-11)


def pin_cache_arithmetic(O):
    """Per-token storage figures printed on the pages."""
    g = json.load(open(os.path.join(GOLDEN, "cache_arithmetic.json")))
    v3, v2 = g["v3"], g["v2"]
    mla = O.cache_values_per_token(v3["d_c"], v3["d_rope"])
    mha = O.mha_values_per_token(v3["heads"], v3["qk_dim"], v3["v_dim"])
    assert mla == v3["mla_values_per_token_layer"]
    assert mha == v3["mha_values_per_token_layer"]
    assert round(mha / mla) == v3["ratio_approx"]
    assert round(mla * 2 * v3["layers"] / 1000) == v3["kb_per_token_approx"]
    assert O.cache_values_per_token(v2["d_c"], v2["d_rope"]) * v2["layers"] == v2["scalars_per_token"]
    assert v2["scalars_per_token"] * 2 / 1024 == v2["kb_per_token_fp16"]


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
