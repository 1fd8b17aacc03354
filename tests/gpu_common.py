"""Shared helpers of the GPU tests: generated inputs, the oracle on sampled
outputs, and the error measure max|gpu - ref| / max|ref|."""
from __future__ import annotations

import functools

import numpy as np
import torch

from mla_latent_kv_43_b200 import inputs as gen
from oracle import mla_oracle as O

# Parity bars: fp32 workloads 1e-5, bf16 workloads 1e-2 (max|d| / max|ref|).
TOL = {"fp32": 1e-5, "bf16": 1e-2}


@functools.lru_cache(maxsize=2)
def host_inputs(name: str):
    return gen.generate(gen.WORKLOADS[name])


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def oracle_out(w, host, batches=None, heads=None):
    if "sel" in host:                       # decode over the selected keys
        k_rot = O.rope_cache(host["k_rope"], host["seq_lens"], w.rope_base)
        return O.decode_sparse(host["q_nope"], host["q_rope"], host["W_uk"], host["W_uv"], host["c_kv"], k_rot,
                               host["seq_lens"], host["sel"].numpy(), host["n_sel"].numpy(), w.n_q,
                               w.softmax_scale, w.rope_base, batches=batches, heads=heads)
    return O.decode_step(host, w.n_q, w.d_c, w.softmax_scale, w.rope_base,
                         batches=batches, heads=heads)


def sampled(arr, batches, heads):
    """arr [B][n_q][H][v] -> the selected (batch, head) entries, stacked."""
    a = np.asarray(arr)
    return np.stack([a[b, :, h] for b in batches for h in heads])


def gpu_out(prob) -> np.ndarray:
    return prob.out.double().cpu().numpy()
