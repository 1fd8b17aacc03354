"""Prefill on the GPU (mla_prefill): the decode's attention evaluated in the
materialised factorisation -- per-head keys and values expanded from the
latent once, then causal attention per head ("Understanding MLA", section 6;
"Multi-Head Latent Attention", section 3).

* against the fp64 oracle (bf16 bar): a whole prompt (every cached token a
  query), chunked prefill behind earlier context, ragged lengths, query
  counts that leave a partial 128-query tile, key counts that leave a partial
  64-key tile, any head count;
* the same inputs through the absorbed decode agree within the bf16 bar;
* NaN in cache slots past a sequence never reaches its outputs;
* a bad length sets MLA_ERR_LEN and zeroes that sequence's outputs only."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from gpu_common import TOL, gpu_out, host_inputs, oracle_out, rel_err, sampled  # noqa: E402
from mla_latent_kv_43_b200 import binding as B  # noqa: E402
from mla_latent_kv_43_b200 import inputs as gen  # noqa: E402
from mla_latent_kv_43_b200.runner import DeviceProblem  # noqa: E402
from oracle import mla_oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

GEOM = dict(d_c=512, d_rope=64, qk_nope=128, v_dim=128)


def _problem(lens, n_q, heads, seed, capacity=None):
    w = gen.tiny("bf16", lens=lens, n_q=n_q, heads=heads, seed=seed, latent_rms_norm=True, prefill=True,
                 capacity=capacity, **GEOM)
    host = gen.generate(w)
    return w, host, DeviceProblem(w, host)


@pytest.mark.parametrize("lens,n_q,heads", [
    ((200,), 200, 2),              # whole prompt: 2 query tiles (128 + 72), 4 key tiles (last partial)
    ((300, 130, 257), 130, 3),     # chunked: 130 new queries behind up to 170 earlier keys
    ((64, 65), 1, 4),              # one query each (a decode step through the prefill path)
    ((129, 128, 127), 127, 2),     # tile edges
])
def test_prefill_matches_oracle(lens, n_q, heads):
    w, host, prob = _problem(lens, n_q, heads, seed=sum(lens) + n_q)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    ref = oracle_out(w, host)
    got = gpu_out(prob)
    err = rel_err(got, ref)
    print(f"lens {lens} n_q {n_q} heads {heads}: {err:.2e}")
    assert err <= TOL["bf16"]


def test_prefill_v3_heads_sampled():
    """128 heads, a 1000-token prompt: sampled heads against the oracle."""
    w, host, prob = _problem((1000,), 1000, 128, seed=41)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    hs = [0, 77, 127]
    ref = oracle_out(w, host, heads=hs)
    err = rel_err(sampled(gpu_out(prob), [0], hs), sampled(ref, [0], hs))
    print(f"v3 1000-token prompt: {err:.2e}")
    assert err <= TOL["bf16"]


def test_prefill_agrees_with_absorbed_decode():
    lens, n_q = (300, 250), 200
    w, host, prob = _problem(lens, n_q, 128, seed=43)
    prob.step()
    dec = DeviceProblem(w.with_(prefill=False), host)
    dec.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0 and dec.get_status() == 0
    err = rel_err(gpu_out(prob), gpu_out(dec))
    print(f"prefill vs absorbed decode: {err:.2e}")
    assert err <= TOL["bf16"]


def test_prefill_nan_past_the_sequence_does_not_leak():
    lens, n_q = (150, 90), 90
    w, host, prob = _problem(lens, n_q, 2, seed=44, capacity=260)
    prob.step()
    torch.cuda.synchronize()
    clean = prob.out.clone()
    for b, L in enumerate(lens):
        prob.cache[b, L:] = float("nan")
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    assert torch.isfinite(prob.out.float()).all()
    assert torch.equal(prob.out, clean)


def test_prefill_bad_length_zeroes_that_sequence():
    lens, n_q = (150, 90, 120), 90
    w, host, prob = _problem(lens, n_q, 2, seed=45)
    bad = host["seq_lens"].clone()
    bad[1] = n_q - 1                        # fewer keys than queries
    prob.seq_lens.copy_(bad)
    prob.out.fill_(1.0)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == B.CODES["MLA_ERR_LEN"]
    out = prob.out.float().cpu()
    assert torch.count_nonzero(out[1]) == 0
    ref = oracle_out(w, host, batches=[0, 2])
    got = gpu_out(prob)
    assert rel_err(got[[0, 2]], ref[[0, 2]]) <= TOL["bf16"]


def test_prefill_workload_sampled():
    """The benchmarked 4096-token prompt, sampled heads."""
    w = gen.WORKLOADS["v3_b1_prefill4096"]
    host = host_inputs(w.name)
    prob = DeviceProblem(w, host)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    hs = [0, 127]
    ref = oracle_out(w, host, heads=hs)
    err = rel_err(sampled(gpu_out(prob), [0], hs), sampled(ref, [0], hs))
    print(f"v3_b1_prefill4096: {err:.2e}")
    assert err <= TOL["bf16"]
