"""Algorithmic bytes and FLOPs of one decode step (what the roofline divides).

Storage per cached token and layer is the latent plus the rope key, d_c +
d_rope values ("Understanding MLA (Multi-head Latent Attention)", section 5:
512 + 64 = 576; at 2 bytes that is 1152 B, and over DeepSeek-V3's 61 layers
about 70 KB per token, as the akshathtiwari "MLA" blog states).

Counting rules: every cache row a query can see is read once per sequence
(all heads and all query tokens of a sequence share it); each weight is read
once per step; queries are read and outputs written once.  Split-KV partial
results are implementation traffic and are not counted.  FLOPs are 2 per
multiply-add of the absorbed form: per visible key and query token,
H * (d_c + d_rope) for the score and H * d_c for the weighted latent sum;
per query token, H * qk_nope * d_c for the absorption and H * d_c * v_dim
for the value up-projection; 2 * hidden * (d_c + d_rope) per appended token;
2 * H * v_dim * hidden_out per query token for the output projection, which
reads W_O once and the head outputs once more and writes y.

A prefill workload (the materialised factorisation) counts its own FLOPs:
2 * H * (qk_nope + d_rope + v_dim) per visible (query, key) pair for the
attention and 2 * d_c * H * (qk_nope + v_dim) per cached key for expanding
the latent into per-head keys and values; its bytes are the same inputs and
outputs (the expanded keys and values are implementation traffic).
"""
from __future__ import annotations

import json
import os
from typing import Dict, Sequence

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def cache_bytes_per_token(d_c: int, d_rope: int, elem_bytes: int, layers: int = 1) -> int:
    return (d_c + d_rope) * elem_bytes * layers


def load_peaks() -> Dict[str, float]:
    """Measured peaks of this GPU pool, else the recorded fallback figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def step_work(w, lens: Sequence[int]) -> Dict[str, float]:
    """Algorithmic bytes/FLOPs of one step of workload ``w`` with lengths ``lens``."""
    es = 4 if w.dtype == "fp32" else 2
    D = w.d_c + w.d_rope
    H = w.heads
    B = w.batch
    qt = B * w.n_q                                     # query tokens
    keys_per_seq = [int(L) for L in lens]
    visible = sum(sum(L - w.n_q + j + 1 for j in range(w.n_q)) for L in keys_per_seq)
    r = {}
    r["cache_bytes"] = sum(keys_per_seq) * D * es
    if w.top_k:
        # sparse decode: each query reads only its selected rows (min(k, p + 1) of them)
        visible = sum(sum(min(w.top_k, L - w.n_q + j + 1) for j in range(w.n_q)) for L in keys_per_seq)
        r["cache_bytes"] = visible * D * es
    r["weight_bytes"] = H * w.d_c * (w.qk_nope + w.v_dim) * es
    r["q_bytes"] = qt * H * (w.qk_nope + w.d_rope) * es
    r["out_bytes"] = qt * H * w.v_dim * es
    r["core_flops"] = visible * 2 * H * (D + w.d_c)
    r["proj_flops"] = qt * 2 * H * w.d_c * (w.qk_nope + w.v_dim)
    if w.prefill:
        r["core_flops"] = visible * 2 * H * (w.qk_nope + w.d_rope + w.v_dim)
        r["proj_flops"] = sum(keys_per_seq) * 2 * w.d_c * H * (w.qk_nope + w.v_dim)
    r["append_bytes"] = 0
    r["append_flops"] = 0
    if w.n_new:
        m = B * w.n_new
        r["append_bytes"] = (w.hidden * D + m * w.hidden + m * D) * es
        r["append_flops"] = 2 * m * w.hidden * D
    r["oproj_bytes"] = 0
    r["oproj_flops"] = 0
    if w.hidden_out:
        K = H * w.v_dim
        r["oproj_bytes"] = (K * w.hidden_out + qt * K + qt * w.hidden_out) * es
        r["oproj_flops"] = 2 * qt * K * w.hidden_out
    r["bytes"] = (r["cache_bytes"] + r["weight_bytes"] + r["q_bytes"] + r["out_bytes"] + r["append_bytes"]
                  + r["oproj_bytes"])
    r["flops"] = r["core_flops"] + r["proj_flops"] + r["append_flops"] + r["oproj_flops"]
    r["query_tokens"] = qt
    return r


def kernel_bytes(kernel: str, w, lens: Sequence[int], q_lat_elem: int, o_lat_elem: int) -> float:
    """Algorithmic bytes of one launch of a kernel of the step.

    The attention kernel's are the cache rows it must read, once per sequence
    (what the method's compressed cache shrinks); its absorbed queries in and
    latent outputs out are workspace intermediates, counted separately by
    kernel_intermediate_bytes.  Absorb/up-projection move their weight and
    activations; append moves W_dkv, x and the new rows.
    """
    es = 4 if w.dtype == "fp32" else 2
    D = w.d_c + w.d_rope
    qt = w.batch * w.n_q
    H = w.heads
    if "prefill" in kernel:
        return 0.0                     # tensor-bound: see kernel_flops
    if "attend" in kernel or "core" in kernel:
        keys = sum(int(L) for L in lens)
        if w.top_k:
            keys = sum(sum(min(w.top_k, int(L) - w.n_q + j + 1) for j in range(w.n_q)) for L in lens)
        return keys * D * es
    if "absorb" in kernel:
        return H * w.d_c * w.qk_nope * es + qt * H * (w.qk_nope + w.d_rope) * es + qt * H * D * q_lat_elem
    if "upproj" in kernel:
        return H * w.d_c * w.v_dim * es + qt * H * w.d_c * o_lat_elem + qt * H * w.v_dim * es
    if "append" in kernel:
        m = w.batch * w.n_new
        return (w.hidden * D + m * w.hidden + m * D) * es
    if "oproj" in kernel:
        K = H * w.v_dim
        return (K * w.hidden_out + qt * K + qt * w.hidden_out) * es
    return 0.0


def visible_pairs(w, lens: Sequence[int]) -> int:
    """(query, key) pairs of a causal step: query j of a sequence of L keys sees
    keys 0 .. L - n_q + j."""
    n = w.n_q
    return sum(n * (int(L) - n + 1) + n * (n - 1) // 2 for L in lens)


def kernel_flops(kernel: str, w, lens: Sequence[int]) -> float:
    """Algorithmic FLOPs of one launch of a tensor-bound kernel (the prefill's
    attention and latent expansion); 0 for the HBM-bound kernels."""
    H = w.heads
    if "prefill_attend" in kernel:
        return 2.0 * H * (w.qk_nope + w.d_rope + w.v_dim) * visible_pairs(w, lens)
    if "prefill_expand" in kernel:
        return 2.0 * sum(int(L) for L in lens) * w.d_c * H * (w.qk_nope + w.v_dim)
    return 0.0


def kernel_intermediate_bytes(kernel: str, w, q_lat_elem: int, o_lat_elem: int) -> float:
    """Workspace intermediates a launch moves besides its algorithmic bytes:
    for the attention kernel, the absorbed queries read and the weighted
    latents written (split-KV partials not included)."""
    if "attend" in kernel or "core" in kernel:
        qt = w.batch * w.n_q
        return qt * w.heads * (w.d_c + w.d_rope) * q_lat_elem + qt * w.heads * w.d_c * o_lat_elem
    return 0.0
