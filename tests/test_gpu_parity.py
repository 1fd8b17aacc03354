"""CUDA path against the fp64 oracle on the five workloads and the top-k
sparse workload (same seeded inputs, in the launch configuration the
benchmark times).  Every (batch, head) output row is compared for the tiny
workload, the batched headline workload and the append workload; the
single-sequence and top-k workloads compare sampled (batch, head) rows."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from gpu_common import TOL, gpu_out, host_inputs, oracle_out, rel_err, sampled  # noqa: E402
from mla_latent_kv_43_b200 import inputs as gen  # noqa: E402
from mla_latent_kv_43_b200.runner import DeviceProblem  # noqa: E402

pytestmark = pytest.mark.gpu

# (workload, sampled batches or None for all, sampled heads or None for all)
CASES = [
    ("tiny_fp32", None, None),
    ("v3_b1_ctx8192", [0], list(range(0, 128, 4))),
    ("v3_b64_ragged", None, None),
    ("v3_b4_ctx131072", [0, 3], [0, 64, 127]),
    ("v3_b32_append2", None, None),
    ("v3_b32_topk2048", [0, 17, 31], [0, 64, 127]),
]


@pytest.mark.parametrize("name,batches,heads", CASES, ids=[c[0] for c in CASES])
def test_workload_parity(name, batches, heads):
    w = gen.WORKLOADS[name]
    host = host_inputs(name)
    prob = DeviceProblem(w, host)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    got = gpu_out(prob)
    assert np.isfinite(got).all()
    bs = list(range(w.batch)) if batches is None else batches
    hs = list(range(w.heads)) if heads is None else heads
    ref = oracle_out(w, host, batches=bs, heads=hs)
    err = rel_err(sampled(got, bs, hs), sampled(ref, bs, hs))
    print(f"{name}: max|d|/max|ref| = {err:.3e}")
    assert err <= TOL[w.dtype], err


@pytest.mark.parametrize("splits", [1, 2, 7])
def test_tiny_split_count_invariance(splits):
    w = gen.WORKLOADS["tiny_fp32"]
    host = host_inputs("tiny_fp32")
    prob = DeviceProblem(w, host, splits=splits)
    prob.step()
    assert prob.get_status() == 0
    ref = oracle_out(w, host)
    assert rel_err(gpu_out(prob), ref) <= TOL["fp32"]
