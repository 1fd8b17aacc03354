"""Seeded synthetic inputs for MLA absorbed decode.

This module only draws random numbers, shapes their distribution and casts
them to the storage dtype.  It holds none of the attention arithmetic, so both
the CUDA path and the fp64 oracle can be fed from it without sharing any of
the method's code.

Geometry follows DeepSeek-V3 as stated on "Understanding MLA (Multi-head
Latent Attention)", section 3 (hidden 7168, 128 heads, latent 512, rope key 64,
query/key width 192 = 128 + 64, value width 128) and on "Multi-Head Latent
Attention", section 4 ("Carry-over to V3": d_c = 512, d_R = 64, 61 layers).

Draw order (one numpy PCG64 stream per workload, seeded with ``seed``):
lens (only when drawn), q_nope, q_rope, c_kv, k_rope, W_uk, W_uv, x, W_dkv.
Every draw is ``standard_normal(dtype=float32)``; a weight "~ N(0, 1/n)" is the
draw times ``1/sqrt(n)``; an "RMS-normalised latent" row is the draw divided
by the root mean square of that row.  The cast to the storage dtype happens
once, at the end; those stored values are what both sides see.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode problem.

    ``lens`` are the per-sequence key counts *including* the query tokens'
    own cache entries; query j of sequence b sits at position
    ``lens[b] - n_q + j``.  When ``n_new`` > 0 the last ``n_new`` entries of
    every sequence are produced by the append step from ``x`` and ``W_dkv``
    rather than drawn.
    """

    name: str
    dtype: str                      # "fp32" or "bf16": storage and I/O dtype
    batch: int
    heads: int
    d_c: int
    d_rope: int
    qk_nope: int
    v_dim: int
    n_q: int
    lens: Optional[Tuple[int, ...]]  # None -> drawn uniformly in lens_range
    capacity: int
    lens_range: Optional[Tuple[int, int]] = None   # inclusive bounds
    latent_rms_norm: bool = False
    hidden: int = 0
    n_new: int = 0
    top_k: int = 0                  # > 0: each query attends a selected subset of its keys
    hidden_out: int = 0             # > 0: the step ends with the output projection to this width
    prefill: bool = False           # True: the materialised factorisation (mla_prefill)
    rope_base: float = 10000.0
    seed: int = 0

    @property
    def d(self) -> int:
        return self.d_c + self.d_rope

    @property
    def softmax_scale(self) -> float:
        # The scale uses the full query/key width qk_nope + d_rope
        # ("Understanding MLA", Phase D, step D2: divide by sqrt(192)).
        return 1.0 / math.sqrt(self.qk_nope + self.d_rope)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


V3 = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128)

# The five workloads, in the order the headline configuration list gives them.
WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload(
        name="tiny_fp32", dtype="fp32", batch=2, heads=4, d_c=64, d_rope=16,
        qk_nope=32, v_dim=32, n_q=1, lens=(37, 100), capacity=100, seed=0),
    "v3_b1_ctx8192": Workload(
        name="v3_b1_ctx8192", dtype="bf16", batch=1, n_q=1, lens=(8192,),
        capacity=8192, latent_rms_norm=True, seed=1, **V3),
    "v3_b64_ragged": Workload(
        name="v3_b64_ragged", dtype="bf16", batch=64, n_q=1, lens=None,
        lens_range=(1024, 4096), capacity=4096, latent_rms_norm=True, seed=2,
        **V3),
    "v3_b4_ctx131072": Workload(
        name="v3_b4_ctx131072", dtype="bf16", batch=4, n_q=1,
        lens=(131072,) * 4, capacity=131072, latent_rms_norm=True, seed=3,
        **V3),
    "v3_b32_append2": Workload(
        name="v3_b32_append2", dtype="bf16", batch=32, n_q=2,
        lens=(4098,) * 32, capacity=4098, latent_rms_norm=True, hidden=7168,
        n_new=2, seed=4, **V3),
    # sparse decode over a top-k selection of the cached keys ("Multi-Head
    # Latent Attention", section 4: k = 2048 per query); the selection is a
    # seeded uniform subset of the visible keys, standing in for an indexer
    "v3_b32_topk2048": Workload(
        name="v3_b32_topk2048", dtype="bf16", batch=32, n_q=1, lens=(8192,) * 32,
        capacity=8192, latent_rms_norm=True, top_k=2048, seed=5, **V3),
    # the batched decode followed by the output projection W_O to the model
    # width 7168 ("Understanding MLA", Phase D step D2); same draws as
    # v3_b64_ragged plus W_O
    "v3_b64_ragged_oproj": Workload(
        name="v3_b64_ragged_oproj", dtype="bf16", batch=64, n_q=1, lens=None,
        lens_range=(1024, 4096), capacity=4096, latent_rms_norm=True, seed=2,
        hidden_out=7168, **V3),
    # prefill of a 4096-token prompt (every cached token is a query, causal)
    # in the materialised factorisation ("Understanding MLA", section 6:
    # training / prefill expands the latent and runs ordinary attention)
    "v3_b1_prefill4096": Workload(
        name="v3_b1_prefill4096", dtype="bf16", batch=1, n_q=4096, lens=(4096,),
        capacity=4096, latent_rms_norm=True, prefill=True, seed=6, **V3),
}
WORKLOAD_ORDER = list(WORKLOADS)


def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _rms_rows(a: np.ndarray) -> np.ndarray:
    """Divide every row (last axis) by its root mean square (input shaping)."""
    for i in range(a.shape[0]):            # row blocks keep the temporaries small
        blk = a[i]
        rms = np.sqrt(np.mean(blk.astype(np.float64) ** 2, axis=-1, keepdims=True))
        a[i] = (blk / rms).astype(np.float32)
    return a


def _cast(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype)


def generate(w: Workload) -> Dict[str, torch.Tensor]:
    """Draw one workload's inputs as CPU tensors in the storage dtype.

    Returns q_nope [B][n_q][H][qk_nope], q_rope [B][n_q][H][d_rope] (not yet
    rotated), c_kv [B][cap][d_c], k_rope [B][cap][d_rope] (not yet rotated),
    W_uk [H][d_c][qk_nope], W_uv [H][d_c][v_dim], seq_lens int32 [B]; with
    n_new > 0 also x [B*n_new][hidden], W_dkv [hidden][d_c+d_rope],
    positions int32 [B*n_new] and old_lens int32 [B]; with top_k > 0 also
    sel int32 [B][n_q][top_k] (distinct visible slots, unused tail entries 0)
    and n_sel int32 [B][n_q] = min(top_k, p + 1); with hidden_out > 0 also
    W_O [H*v_dim][hidden_out] (drawn last, so the other draws do not change).
    """
    rng = np.random.default_rng(w.seed)
    if w.lens is None:
        lo, hi = w.lens_range
        lens = rng.integers(lo, hi + 1, size=w.batch).astype(np.int32)
    else:
        lens = np.asarray(w.lens, dtype=np.int32)
    assert lens.shape == (w.batch,) and int(lens.max()) <= w.capacity
    assert int(lens.min()) >= w.n_q
    dt = w.torch_dtype
    out: Dict[str, torch.Tensor] = {}
    out["q_nope"] = _cast(_normal(rng, (w.batch, w.n_q, w.heads, w.qk_nope)), dt)
    out["q_rope"] = _cast(_normal(rng, (w.batch, w.n_q, w.heads, w.d_rope)), dt)
    c = _normal(rng, (w.batch, w.capacity, w.d_c))
    if w.latent_rms_norm:
        c = _rms_rows(c)
    out["c_kv"] = _cast(c, dt)
    del c
    out["k_rope"] = _cast(_normal(rng, (w.batch, w.capacity, w.d_rope)), dt)
    wstd = 1.0 / math.sqrt(w.d_c)
    out["W_uk"] = _cast(_normal(rng, (w.heads, w.d_c, w.qk_nope), wstd), dt)
    out["W_uv"] = _cast(_normal(rng, (w.heads, w.d_c, w.v_dim), wstd), dt)
    out["seq_lens"] = torch.from_numpy(lens.copy())
    if w.n_new:
        m = w.batch * w.n_new
        out["x"] = _cast(_normal(rng, (m, w.hidden)), dt)
        out["W_dkv"] = _cast(_normal(rng, (w.hidden, w.d), 1.0 / math.sqrt(w.hidden)), dt)
        old = lens - w.n_new
        pos = (old[:, None] + np.arange(w.n_new, dtype=np.int32)[None, :]).reshape(-1)
        out["positions"] = torch.from_numpy(pos.astype(np.int32))
        out["old_lens"] = torch.from_numpy(old.astype(np.int32))
    if w.top_k:
        sel = np.zeros((w.batch, w.n_q, w.top_k), dtype=np.int32)
        n_sel = np.zeros((w.batch, w.n_q), dtype=np.int32)
        for b in range(w.batch):
            for j in range(w.n_q):
                p = int(lens[b]) - w.n_q + j
                n = min(w.top_k, p + 1)
                sel[b, j, :n] = rng.choice(p + 1, size=n, replace=False)
                n_sel[b, j] = n
        out["sel"] = torch.from_numpy(sel)
        out["n_sel"] = torch.from_numpy(n_sel)
    if w.hidden_out:
        K = w.heads * w.v_dim
        out["W_O"] = _cast(_normal(rng, (K, w.hidden_out), 1.0 / math.sqrt(K)), dt)
    return out


def tiny(dtype: str = "fp32", *, batch=None, heads=3, d_c=8, d_rope=4, qk_nope=6,
         v_dim=5, n_q=1, lens=(5, 9), capacity=None, seed=0, latent_rms_norm=False,
         hidden=0, n_new=0, top_k=0, hidden_out=0, prefill=False) -> Workload:
    """A small custom workload for pins and edge cases (batch = len(lens))."""
    cap = capacity if capacity is not None else max(lens)
    if batch is None:
        batch = len(lens)
    return Workload(name="custom", dtype=dtype, batch=batch, heads=heads, d_c=d_c,
                    d_rope=d_rope, qk_nope=qk_nope, v_dim=v_dim, n_q=n_q,
                    lens=tuple(lens), capacity=cap, latent_rms_norm=latent_rms_norm,
                    hidden=hidden, n_new=n_new, top_k=top_k, hidden_out=hidden_out, prefill=prefill,
                    seed=seed)


def sharpen(host: Dict[str, torch.Tensor], *, gain: int = 4, late=None, late_gain: int = 2,
            dominant=None, dominant_gain: int = 4, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Reshape generated inputs into a large-score, peaky-softmax case.

    * ``W_uk[h]`` becomes a signed selection times ``gain``: latent row i of
      head h holds +-gain at one q_nope column (a seeded permutation, every
      column used d_c / qk_nope times) and zeros elsewhere, so each absorbed
      query entry is +-gain times one stored q_nope value -- exactly
      representable in the storage dtype when ``gain`` is a power of two;
    * ``q_rope`` is multiplied by ``gain``;
    * the cache rows ``late[b] = (lo, hi)`` of sequence b (latent and raw rope
      key) are multiplied by ``late_gain``, and row ``dominant[b]`` by
      ``dominant_gain``.

    With power-of-two gains every reshaped value is the stored value times a
    power of two, so no rounding is added.  Returns a new dict; ``host`` is
    left unchanged.
    """
    for g in (gain, late_gain, dominant_gain):
        assert g > 0 and (g & (g - 1)) == 0, "gains must be powers of two"
    out = dict(host)
    H, d_c, qk = host["W_uk"].shape
    assert d_c % qk == 0
    rng = np.random.default_rng(seed)
    W = np.zeros((H, d_c, qk), dtype=np.float32)
    for h in range(H):
        cols = rng.permutation(np.repeat(np.arange(qk), d_c // qk))
        signs = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=d_c)
        W[h, np.arange(d_c), cols] = signs * gain
    out["W_uk"] = _cast(W, host["W_uk"].dtype)
    out["q_rope"] = host["q_rope"] * gain
    c, kr = host["c_kv"].clone(), host["k_rope"].clone()
    for b in range(c.shape[0]):
        if late is not None and late[b] is not None:
            lo, hi = late[b]
            c[b, lo:hi] *= late_gain
            kr[b, lo:hi] *= late_gain
        if dominant is not None and dominant[b] is not None:
            c[b, dominant[b]] *= dominant_gain
            kr[b, dominant[b]] *= dominant_gain
    out["c_kv"], out["k_rope"] = c, kr
    return out
