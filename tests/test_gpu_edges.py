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


def _scaled_scores(w, host, b, h):
    """Scaled scores of query (b, last) head h against its visible keys (fp64,
    from the oracle's absorbed query and rotated cache keys)."""
    L = int(host["seq_lens"][b])
    p = L - w.n_q + (w.n_q - 1)
    q = O.absorbed_query(host["q_nope"][b, -1, h].double().numpy(), host["q_rope"][b, -1, h].double().numpy(),
                         host["W_uk"][h].double().numpy(), p, w.rope_base)
    k_rot = O.rope_cache(host["k_rope"][b:b + 1, :L].double().numpy(), [L], w.rope_base)[0]
    K = np.concatenate([host["c_kv"][b, :L].double().numpy(), k_rot], axis=1)
    return (K @ q) * w.softmax_scale


def test_large_logits_peaky_softmax_many_pieces():
    """Tensor-core path with scaled scores spanning more than +-40, a handful of
    keys holding most of each head's softmax weight, a row maximum that grows
    by more than 2^8 (base 2) late in the sequence, and each sequence cut into
    many split-KV pieces, every (batch, head) row compared at the bf16 bar.
    The absorbed query is exactly representable in bf16 (a signed selection
    of q_nope times a power of two), so the comparison measures the kernel's
    own arithmetic rather than the rounding of the query, whose effect grows
    with the score magnitude for any bf16-operand kernel.  ("Understanding
    MLA", Phase D step D2: softmax(Q K^T / sqrt(192)) V.)"""
    lens = (8192, 2600)
    w, host = make("bf16_v3", lens=lens, capacity=8192, seed=11)
    late = [(lens[0] - 700, lens[0] - 600), (lens[1] - 300, lens[1] - 200)]
    host = gen.sharpen(host, gain=4, late=late, late_gain=2, dominant=[1000, 100], dominant_gain=4, seed=12)
    # the inputs are what the docstring says (checked on a few heads, fp64)
    grew, span = 0, 0.0
    for h in (0, 37, 64, 90):
        s = _scaled_scores(w, host, 0, h)
        span = max(span, float(np.abs(s).max()))
        wts = np.exp(s - s.max())
        wts /= wts.sum()
        assert np.sort(wts)[-8:].sum() > 0.5
        l2 = s * np.log2(np.e)
        grew += l2[late[0][0]:].max() > l2[: late[0][0]].max() + 8
    assert span > 40 and grew >= 1, (span, grew)
    splits = 48
    prob = DeviceProblem(w, host, splits=splits)
    assert prob.layout["splits"] == splits
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    got = gpu_out(prob)
    assert np.isfinite(got).all()
    ref = oracle_out(w, host)
    err = rel_err(got, ref)
    print(f"large logits: max|d|/max|ref| = {err:.3e}")
    assert err <= TOL["bf16"], err


def test_one_sequence_in_74_pieces():
    """One 32768-key sequence cut into 74 split-KV pieces (one per cluster of
    the B200's 148 SMs): the log-sum-exp merge of many pieces per token."""
    w, host = make("bf16_v3", lens=(32768,), capacity=32768, seed=13)
    prob = DeviceProblem(w, host, splits=74)
    assert prob.layout["splits"] == 74
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    hs = list(range(0, 128, 8))
    ref = oracle_out(w, host, batches=[0], heads=hs)
    err = rel_err(sampled(gpu_out(prob), [0], hs), sampled(ref, [0], hs))
    assert err <= TOL["bf16"], err


def test_plan_for_many_query_tokens():
    """More query tokens than the staged key-tile plan holds (600 > 512): the
    plan takes its general path; every sequence is short and ragged, so most
    clusters hold many whole tokens and the boundaries cut a few."""
    rng = np.random.default_rng(17)
    lens = tuple(int(x) for x in rng.integers(1, 300, size=600))
    w, host = make("bf16_v3", lens=lens, capacity=300, seed=17)
    prob = DeviceProblem(w, host)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    bs = [0, 1, 255, 256, 511, 512, 513, 599]
    check(w, host, prob, batches=bs)
