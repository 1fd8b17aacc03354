"""The append step on the GPU: exactly the addressed cache slots change
(bit-exact slot indexing against a sentinel pattern), their values match the
oracle's fp64 rows, and positions outside the cache set MLA_ERR_POS."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from gpu_common import TOL, rel_err  # noqa: E402
from mla_latent_kv_43_b200 import binding as B  # noqa: E402
from mla_latent_kv_43_b200 import inputs as gen  # noqa: E402
from oracle import mla_oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

SMALL = dict(heads=2, d_c=8, d_rope=4, qk_nope=6, v_dim=5)
V3 = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128)
CASES = {"fp32_small": ("fp32", SMALL, 24), "bf16_small": ("bf16", SMALL, 40),
         "bf16_v3": ("bf16", V3, 7168)}


def run_append(case, positions, batch, n_new, capacity, seed=0, gamma=None):
    dtype, g, hidden = CASES[case]
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    rng = np.random.default_rng(seed)
    D = g["d_c"] + g["d_rope"]
    x = torch.from_numpy(rng.standard_normal((batch * n_new, hidden), dtype=np.float32)).to(tdt)
    W = torch.from_numpy((rng.standard_normal((hidden, D), dtype=np.float32) / np.sqrt(hidden)).astype(np.float32)).to(tdt)
    # sentinel: a fixed byte pattern that is a finite value in both dtypes
    cache = torch.empty(batch, capacity, D, dtype=tdt, device="cuda")
    cache.view(torch.uint8).fill_(0x3C)
    before = cache.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dims = B.make_dims(dtype=dtype, **g)
    pos = torch.tensor(positions, dtype=torch.int32)
    g = None if gamma is None else torch.as_tensor(gamma, dtype=torch.float32).cuda()
    B.mla_append(dims, x.cuda(), W.cuda(), pos.cuda(), cache, status, batch=batch, n_new=n_new, rms_gamma=g)
    code = B.mla_get_status(status)
    return dims, x, W, pos, before, cache, code


@pytest.mark.parametrize("case", list(CASES))
def test_append_writes_exactly_the_addressed_slots(case):
    batch, n_new, cap = 3, 2, 70
    positions = [5, 6, 0, 1, cap - 2, cap - 1]
    dims, x, W, pos, before, cache, code = run_append(case, positions, batch, n_new, cap, seed=1)
    assert code == 0
    changed = (cache.view(torch.int16 if cache.element_size() == 2 else torch.int32)
               != before.view(torch.int16 if cache.element_size() == 2 else torch.int32)).any(-1).cpu()
    expect = torch.zeros(batch, cap, dtype=torch.bool)
    for r, p in enumerate(positions):
        expect[r // n_new, p] = True
    assert torch.equal(changed, expect)
    rows = O.append_rows(x, W, positions, dims.d_c, dims.rope_base)
    got = np.stack([cache[r // n_new, p].double().cpu().numpy() for r, p in enumerate(positions)])
    tol = TOL["fp32"] if case.startswith("fp32") else TOL["bf16"]
    assert rel_err(got, rows) <= tol


@pytest.mark.parametrize("case", list(CASES))
def test_append_rejects_positions_outside_the_cache(case):
    batch, n_new, cap = 2, 2, 16
    positions = [3, -1, cap, 15]
    dims, x, W, pos, before, cache, code = run_append(case, positions, batch, n_new, cap, seed=2)
    assert code == B.CODES["MLA_ERR_POS"]
    rows = O.append_rows(x, W, positions, dims.d_c, dims.rope_base)
    same = lambda b, p: torch.equal(cache[b, p], before[b, p])
    assert not same(0, 3) and not same(1, 15)
    # every other slot keeps the sentinel
    mask = torch.ones(batch, cap, dtype=torch.bool)
    mask[0, 3] = mask[1, 15] = False
    assert torch.equal(cache[mask], before[mask])
    tol = TOL["fp32"] if case.startswith("fp32") else TOL["bf16"]
    assert rel_err(cache[0, 3].double().cpu().numpy(), rows[0]) <= tol
    assert rel_err(cache[1, 15].double().cpu().numpy(), rows[3]) <= tol


@pytest.mark.parametrize("hidden", [256, 7168])
@pytest.mark.parametrize("tokens", [1, 37, 300])
def test_tensor_core_append_shapes(hidden, tokens):
    """DeepSeek-V3 latent/rope widths (the tensor-core append): fewer K blocks
    than the cluster's CTAs (hidden 256), a single token, a ragged token count
    and more tokens than one launch tile (300 > 256); every slot written once,
    the rest untouched."""
    CASES["bf16_v3_h"] = ("bf16", V3, hidden)
    try:
        batch, n_new, cap = tokens, 1, 9
        rng = np.random.default_rng(tokens + hidden)
        positions = [int(p) for p in rng.integers(0, cap, size=tokens)]
        dims, x, W, pos, before, cache, code = run_append("bf16_v3_h", positions, batch, n_new, cap, seed=3)
    finally:
        del CASES["bf16_v3_h"]
    assert code == 0
    changed = (cache.view(torch.int16) != before.view(torch.int16)).any(-1).cpu()
    expect = torch.zeros(batch, cap, dtype=torch.bool)
    for r, p in enumerate(positions):
        expect[r, p] = True
    assert torch.equal(changed, expect)
    rows = O.append_rows(x, W, positions, dims.d_c, dims.rope_base)
    got = np.stack([cache[r, p].double().cpu().numpy() for r, p in enumerate(positions)])
    assert rel_err(got, rows) <= TOL["bf16"]


@pytest.mark.parametrize("case", list(CASES))
def test_append_rms_norm_of_the_latent(case):
    """rms_gamma: the latent alone is RMS-normalised before it is cached
    ("Understanding MLA", Phase A step A2); the rope key is bit-identical to the
    un-normalised append; other slots keep the sentinel; a position outside the
    cache still sets MLA_ERR_POS and leaves its slot alone."""
    batch, n_new, cap = 3, 2, 12
    positions = [5, 6, 0, 1, 10, cap]                   # the last one is outside
    dtype, g, hidden = CASES[case]
    gamma = np.random.default_rng(5).uniform(0.5, 2.0, g["d_c"]).astype(np.float32)
    dims, x, W, pos, before, cache, code = run_append(case, positions, batch, n_new, cap, seed=4, gamma=gamma)
    _, _, _, _, _, plain, _ = run_append(case, positions, batch, n_new, cap, seed=4)
    assert code == B.CODES["MLA_ERR_POS"]
    d_c = dims.d_c
    rows = O.append_rows(x, W, positions, d_c, dims.rope_base, rms_gamma=gamma)
    valid = [(r, p) for r, p in enumerate(positions) if p < cap]
    got = np.stack([cache[r // n_new, p].double().cpu().numpy() for r, p in valid])
    ref = np.stack([rows[r] for r, _ in valid])
    tol = TOL["fp32"] if case.startswith("fp32") else TOL["bf16"]
    assert rel_err(got[:, :d_c], ref[:, :d_c]) <= tol
    for r, p in valid:
        assert torch.equal(cache[r // n_new, p, d_c:], plain[r // n_new, p, d_c:])
    mask = torch.ones(batch, cap, dtype=torch.bool)
    for r, p in valid:
        mask[r // n_new, p] = False
    assert torch.equal(cache[mask], before[mask])
