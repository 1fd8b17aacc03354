"""mla_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (it runs in the library's fixed scratch area instead of a
caller-provided workspace).  Its output must match mla_decode's on the same
inputs, on two calls in a row (the second call reuses whatever the first left
in the shared scratch, and after a different problem ran through it), and an
oversized request must be refused on the host.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import ctypes
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from gpu_common import TOL, rel_err  # noqa: E402
from mla_latent_kv_43_b200 import binding as B  # noqa: E402
from mla_latent_kv_43_b200 import inputs as gen  # noqa: E402
from mla_latent_kv_43_b200.runner import DeviceProblem  # noqa: E402

pytestmark = pytest.mark.gpu

V3 = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128)
SMALL = dict(heads=3, d_c=8, d_rope=4, qk_nope=6, v_dim=5)
# (dtype, geometry, lens, n_q, splits) of the problem checked, then of a
# different problem run through the same scratch in between: other lengths,
# query count and split count, so the scratch regions (query slices, tile
# plan, partial outputs) sit at other offsets and hold other values
CASES = [("bf16", V3, (130, 67, 200), 1, 4, (300, 5, 77, 1000), 2, 7),
         ("bf16", V3, (64, 131), 2, 2, (513,), 1, 3),
         ("fp32", SMALL, (7, 40, 129), 2, 3, (90, 3), 1, 5)]


def _problem(dtype, geom, lens, n_q, splits, seed):
    w = gen.tiny(dtype, lens=lens, n_q=n_q, seed=seed, latent_rms_norm=(geom is V3), **geom)
    prob = DeviceProblem(w, gen.generate(w), splits=splits)
    assert B.mla_decode_workspace_bytes(prob.dims, w.batch, n_q, prob.max_len, splits) <= B.NOALLOC_SCRATCH_BYTES
    prob.decode()
    assert prob.get_status() == 0
    return prob, prob.out.double().cpu().numpy()


def _noalloc(prob, splits):
    out = torch.full_like(prob.out, float("nan"))
    B.mla_decode_noalloc(prob.dims, prob.q_nope, prob.q_rope, prob.W_uk, prob.W_uv, prob.cache,
                         prob.seq_lens, prob.max_len, out, prob.status, splits)
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    return out.double().cpu().numpy()


@pytest.mark.parametrize("dtype,geom,lens,n_q,splits,lens2,n_q2,splits2", CASES,
                         ids=["v3_nq1", "v3_nq2", "fp32_small"])
def test_noalloc_matches_workspace_decode(dtype, geom, lens, n_q, splits, lens2, n_q2, splits2):
    """Two calls in a row, then a different problem, then the first again:
    each output matches mla_decode's on the same inputs, so nothing a call
    leaves in the shared scratch leaks into the next."""
    prob, ref = _problem(dtype, geom, lens, n_q, splits, seed=31)
    other, ref2 = _problem(dtype, geom, lens2, n_q2, splits2, seed=32)
    for step, (p, r, sp) in enumerate([(prob, ref, splits), (prob, ref, splits), (other, ref2, splits2),
                                       (prob, ref, splits)]):
        got = _noalloc(p, sp)
        assert np.isfinite(got).all(), step
        assert rel_err(got, r) <= TOL[dtype], (step, rel_err(got, r))


def test_noalloc_checks_arguments_like_mla_decode():
    """Bad dims are refused before anything else, an empty problem returns
    MLA_OK, and a refused call reports no launches."""
    dims = B.make_dims(dtype="bf16", **V3)
    fake = 0x10000
    bad = B.make_dims(dtype="bf16", **dict(V3, heads=0))
    for d in (dims, bad):
        rc = B.lib().mla_decode_noalloc(ctypes.byref(d), 0, 1, None, None, None, None, None, 4096, None,
                                        16, None, 0, None, None)
        assert rc == (B.CODES["MLA_OK"] if d is dims else B.CODES["MLA_ERR_ARG"])
        assert B.lib().mla_last_launch_count() == 0
    rc = B.lib().mla_decode_noalloc(ctypes.byref(dims), 2, -1, fake, fake, fake, fake, fake, 4096, fake,
                                    16, fake, 0, fake, None)
    assert rc == B.CODES["MLA_ERR_ARG"]


def test_noalloc_refuses_requests_beyond_its_scratch():
    dims = B.make_dims(dtype="bf16", **V3)
    batch, n_q, max_len, splits = 64, 2, 4096, 0
    assert B.mla_decode_workspace_bytes(dims, batch, n_q, max_len, splits) > B.NOALLOC_SCRATCH_BYTES
    fake = 0x10000
    rc = B.lib().mla_decode_noalloc(ctypes.byref(dims), batch, n_q, fake, fake, fake, fake, fake, 4096, fake,
                                    max_len, fake, splits, fake, None)
    assert rc == B.CODES["MLA_ERR_WORKSPACE"]
    assert B.lib().mla_last_launch_count() == 0
