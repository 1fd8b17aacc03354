"""The output projection on the GPU (mla_output_projection): the per-head
decode outputs, concatenated, times W_O ("Understanding MLA", Phase D step D2).

* against the oracle's fp64 product: fp32 on CUDA cores, bf16 on tensor cores
  at the V3 widths (16384 -> 7168), with ragged token counts, a hidden width
  that ends in a partial 128-column tile and token counts past one token tile;
* a hidden width that is not a multiple of 8 takes the CUDA-core path;
* guard bytes around y keep their pattern (nothing written past the row ends);
* chained after mla_decode: the decode output projected equals the oracle's
  decode projected."""
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
from oracle import mla_oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

SMALL = dict(heads=3, d_c=8, d_rope=4, qk_nope=6, v_dim=5)
V3 = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128)


def _inputs(dtype, g, tokens, hidden, seed):
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    rng = np.random.default_rng(seed)
    K = g["heads"] * g["v_dim"]
    out = torch.from_numpy(rng.standard_normal((tokens, g["heads"], g["v_dim"]), dtype=np.float32)).to(tdt)
    W = torch.from_numpy(rng.standard_normal((K, hidden), dtype=np.float32) / np.float32(np.sqrt(K))).to(tdt)
    return out, W


def _project(dtype, g, out, W, hidden, guard=0):
    tdt = out.dtype
    dims = B.make_dims(dtype=dtype, **g)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    n = out.shape[0] * hidden
    buf = torch.full((guard + n + guard,), -7.0, dtype=tdt, device="cuda")
    y = buf[guard: guard + n].view(out.shape[0], hidden)
    B.mla_output_projection(dims, out.cuda(), W.cuda(), y, status)
    code = B.mla_get_status(status)
    return code, y, buf


@pytest.mark.parametrize("tokens,hidden", [(1, 7), (5, 24), (37, 130)])
def test_fp32_matches_oracle(tokens, hidden):
    out, W = _inputs("fp32", SMALL, tokens, hidden, seed=tokens)
    code, y, _ = _project("fp32", SMALL, out, W, hidden)
    assert code == 0
    assert rel_err(y.double().cpu().numpy(), O.output_projection(out, W)) <= TOL["fp32"]


@pytest.mark.parametrize("tokens,hidden", [(64, 7168), (5, 7168), (1, 512), (300, 136), (33, 100)])
def test_bf16_v3_widths_match_oracle(tokens, hidden):
    out, W = _inputs("bf16", V3, tokens, hidden, seed=hidden + tokens)
    code, y, buf = _project("bf16", V3, out, W, hidden, guard=64)
    assert code == 0
    err = rel_err(y.double().cpu().numpy(), O.output_projection(out, W))
    print(f"tokens {tokens} hidden {hidden}: {err:.2e}")
    assert err <= TOL["bf16"]
    g = buf.float().cpu()
    assert (g[:64] == -7.0).all() and (g[-64:] == -7.0).all()


def test_chained_after_decode():
    w = gen.tiny("bf16", lens=(130, 67, 200), n_q=2, seed=31, latent_rms_norm=True, **V3)
    host = gen.generate(w)
    prob = DeviceProblem(w, host)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    hidden = 1024
    rng = np.random.default_rng(5)
    W = torch.from_numpy(rng.standard_normal((w.heads * w.v_dim, hidden), dtype=np.float32) / 128.0).to(torch.bfloat16)
    tokens = w.batch * w.n_q
    out = prob.out.reshape(tokens, w.heads, w.v_dim)
    code, y, _ = _project("bf16", V3, out, W, hidden)
    assert code == 0
    ref = O.decode_step(host, w.n_q, w.d_c, w.softmax_scale).reshape(tokens, w.heads, w.v_dim)
    assert rel_err(y.double().cpu().numpy(), O.output_projection(ref, W)) <= TOL["bf16"]


def test_workload_with_output_projection():
    """The benchmarked decode + W_O workload at full size (64 sequences,
    16384 -> 7168), sampled sequences through every head."""
    from gpu_common import host_inputs, oracle_out
    w = gen.WORKLOADS["v3_b64_ragged_oproj"]
    host = host_inputs(w.name)
    prob = DeviceProblem(w, host)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    bs = [0, 31, 63]
    dec = oracle_out(w, host, batches=bs)[bs].reshape(len(bs) * w.n_q, w.heads, w.v_dim)
    ref = O.output_projection(dec, host["W_O"])
    rows = [b * w.n_q + j for b in bs for j in range(w.n_q)]
    got = prob.y[rows].double().cpu().numpy()
    err = rel_err(got, ref)
    print(f"v3_b64_ragged_oproj: {err:.2e}")
    assert err <= TOL["bf16"]
