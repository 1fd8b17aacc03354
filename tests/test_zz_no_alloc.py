"""mla_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (it runs in the library's fixed scratch area instead of a
caller-provided workspace).  Its output must match mla_decode's on the same
inputs, on two calls in a row (the second call reuses whatever the first left
in the shared scratch), and an oversized request must be refused on the host.

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
CASES = [("bf16", V3, (130, 67, 200), 1, 4), ("bf16", V3, (64, 131), 2, 2), ("fp32", SMALL, (7, 40, 129), 2, 3)]


@pytest.mark.parametrize("dtype,geom,lens,n_q,splits", CASES, ids=["v3_nq1", "v3_nq2", "fp32_small"])
def test_noalloc_matches_workspace_decode(dtype, geom, lens, n_q, splits):
    w = gen.tiny(dtype, lens=lens, n_q=n_q, seed=31, latent_rms_norm=(geom is V3), **geom)
    prob = DeviceProblem(w, gen.generate(w), splits=splits)
    assert B.mla_decode_workspace_bytes(prob.dims, w.batch, n_q, prob.max_len, splits) <= B.NOALLOC_SCRATCH_BYTES
    prob.decode()
    assert prob.get_status() == 0
    ref = prob.out.double().cpu().numpy()
    for call in range(2):
        out = torch.full_like(prob.out, float("nan"))
        B.mla_decode_noalloc(prob.dims, prob.q_nope, prob.q_rope, prob.W_uk, prob.W_uv, prob.cache,
                             prob.seq_lens, prob.max_len, out, prob.status, splits)
        torch.cuda.synchronize()
        assert prob.get_status() == 0
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all(), call
        assert rel_err(got, ref) <= TOL[dtype], (call, rel_err(got, ref))


def test_noalloc_refuses_requests_beyond_its_scratch():
    dims = B.make_dims(dtype="bf16", **V3)
    batch, n_q, max_len, splits = 64, 2, 4096, 0
    assert B.mla_decode_workspace_bytes(dims, batch, n_q, max_len, splits) > B.NOALLOC_SCRATCH_BYTES
    fake = 0x10000
    rc = B.lib().mla_decode_noalloc(ctypes.byref(dims), batch, n_q, fake, fake, fake, fake, fake, 4096, fake,
                                    max_len, fake, splits, fake, None)
    assert rc == B.CODES["MLA_ERR_WORKSPACE"]
