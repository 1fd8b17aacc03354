"""Edge cases of the decode path on the GPU, for the CUDA-core geometry
(fp32 and bf16) and the DeepSeek-V3 geometry (bf16 tensor-core path):
ragged lengths around tile boundaries, two causal queries, invalid lengths,
garbage beyond each sequence's length, length == capacity, split counts,
the standalone RoPE kernel and the status word."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from gpu_common import TOL, gpu_out, oracle_out, rel_err, sampled  # noqa: E402
from mla_latent_kv_43_b200 import binding as B  # noqa: E402
from mla_latent_kv_43_b200 import inputs as gen  # noqa: E402
from mla_latent_kv_43_b200.runner import DeviceProblem  # noqa: E402
from oracle import mla_oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

SMALL = dict(heads=3, d_c=8, d_rope=4, qk_nope=6, v_dim=5)
V3 = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128)
GEOMS = {"fp32_small": ("fp32", SMALL), "bf16_small": ("bf16", SMALL), "bf16_v3": ("bf16", V3)}
V3_HEADS = [0, 31, 64, 127]


def make(geom, lens, n_q=1, capacity=None, seed=0):
    dtype, g = GEOMS[geom]
    w = gen.tiny(dtype, lens=lens, n_q=n_q, capacity=capacity, seed=seed,
                 latent_rms_norm=(g is V3), **g)
    return w, gen.generate(w)


def heads_of(w):
    return V3_HEADS if w.heads == 128 else list(range(w.heads))


def check(w, host, prob, batches=None):
    got = gpu_out(prob)
    bs = list(range(w.batch)) if batches is None else batches
    hs = heads_of(w)
    ref = oracle_out(w, host, batches=bs, heads=hs)
    err = rel_err(sampled(got, bs, hs), sampled(ref, bs, hs))
    assert err <= TOL[w.dtype], err
    return got


@pytest.mark.parametrize("geom", list(GEOMS))
def test_ragged_lengths_around_tiles(geom):
    w, host = make(geom, lens=(1, 63, 64, 65, 127, 129, 300), capacity=320, seed=1)
    prob = DeviceProblem(w, host)
    prob.step()
    assert prob.get_status() == 0
    check(w, host, prob)


@pytest.mark.parametrize("geom", list(GEOMS))
def test_two_causal_queries(geom):
    w, host = make(geom, lens=(2, 64, 65, 200), n_q=2, capacity=256, seed=2)
    prob = DeviceProblem(w, host)
    prob.step()
    assert prob.get_status() == 0
    check(w, host, prob)


@pytest.mark.parametrize("geom", list(GEOMS))
def test_invalid_lengths_flag_and_zero(geom):
    w, host = make(geom, lens=(5, 40, 7), capacity=64, seed=3)
    prob = DeviceProblem(w, host, max_len=50)
    prob.seq_lens.copy_(torch.tensor([0, 40, 51], dtype=torch.int32))   # < n_q, ok, > max_len
    prob.step()
    assert prob.get_status() == B.CODES["MLA_ERR_LEN"]
    assert prob.get_status() == 0                                        # read clears it
    got = gpu_out(prob)
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    host2 = dict(host)
    host2["seq_lens"] = torch.tensor([5, 40, 7], dtype=torch.int32)
    check(w, host2, prob, batches=[1])


@pytest.mark.parametrize("geom", list(GEOMS))
def test_garbage_beyond_length_is_never_used(geom):
    w, host = make(geom, lens=(3, 70, 130), capacity=192, seed=4)
    clean = DeviceProblem(w, host)
    clean.step()
    dirty = DeviceProblem(w, host)
    for b, L in enumerate((3, 70, 130)):
        dirty.cache[b, L:] = float("nan")
    dirty.step()
    assert dirty.get_status() == 0
    a, b = gpu_out(clean), gpu_out(dirty)
    assert np.isfinite(b).all()
    assert np.array_equal(a, b)
    check(w, host, dirty)


@pytest.mark.parametrize("geom", list(GEOMS))
def test_length_equals_capacity(geom):
    w, host = make(geom, lens=(128, 128), capacity=128, seed=5)
    prob = DeviceProblem(w, host)
    prob.step()
    assert prob.get_status() == 0
    check(w, host, prob)


@pytest.mark.parametrize("geom", list(GEOMS))
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_split_counts(geom, splits):
    w, host = make(geom, lens=(700, 33, 1500), capacity=1536, seed=6)
    prob = DeviceProblem(w, host, splits=splits)
    prob.step()
    assert prob.get_status() == 0
    check(w, host, prob)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_rope_kernel_matches_oracle(dtype):
    rng = np.random.default_rng(7)
    rows, d = 257, 64
    x = rng.standard_normal((rows, 80)).astype(np.float32)
    pos = rng.integers(0, 131072, size=rows).astype(np.int32)
    pos[:3] = [0, 1, 131071]
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    xt = torch.from_numpy(x).to(tdt)
    dev = xt.cuda()
    dims = B.make_dims(heads=1, d_c=16, d_rope=d, qk_nope=8, v_dim=8, dtype=dtype)
    B.mla_rope(dims, rows, dev, 80, torch.from_numpy(pos).cuda(), offset_elems=16)
    got = dev.double().cpu().numpy()
    ref = O.rope(xt.double().numpy()[:, 16:], pos)
    assert np.array_equal(got[:, :16], xt.double().numpy()[:, :16])
    tol = 2e-6 if dtype == "fp32" else 8e-3
    assert rel_err(got[:, 16:], ref) <= tol
