"""Sparse decode on the GPU (mla_decode_sparse): each query attends a
selected subset of its cached keys ("Multi-Head Latent Attention", section 4:
a top-k selection of the cached latents per query).

* against the oracle's decode over the same selection (bf16 bar), with
  ragged counts, tail tiles and two causal queries;
* selecting every visible key reproduces mla_decode (the dense decode runs
  another kernel, so the two agree within the bf16 bar, and both match the
  oracle's dense decode);
* a count outside 1..min(max_sel, p + 1) sets MLA_ERR_LEN and zeroes that
  query's outputs; a slot past the query's position sets MLA_ERR_INDEX."""
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

V3 = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128)
HEADS = [0, 1, 63, 64, 127]


def _problem(lens, n_q, top_k, seed, splits=0):
    w = gen.tiny("bf16", lens=lens, n_q=n_q, top_k=top_k, seed=seed, latent_rms_norm=True, **V3)
    host = gen.generate(w)
    return w, host, DeviceProblem(w, host, splits=splits)


def _oracle(w, host, sel, n_sel, heads=HEADS):
    k_rot = O.rope_cache(host["k_rope"], host["seq_lens"])
    return O.decode_sparse(host["q_nope"], host["q_rope"], host["W_uk"], host["W_uv"], host["c_kv"], k_rot,
                           host["seq_lens"], sel, n_sel, w.n_q, w.softmax_scale, heads=heads)


@pytest.mark.parametrize("top_k,n_q,splits", [(40, 1, 0), (64, 1, 0), (100, 2, 0), (130, 1, 3), (200, 2, 1)])
def test_sparse_matches_oracle(top_k, n_q, splits):
    w, host, prob = _problem((130, 67, 200, 9), n_q, top_k, seed=top_k + n_q, splits=splits)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    ref = _oracle(w, host, host["sel"].numpy(), host["n_sel"].numpy())
    got = prob.out.double().cpu().numpy()
    err = rel_err(got[:, :, HEADS], ref[:, :, HEADS])
    print(f"top_k {top_k} n_q {n_q} splits {splits}: {err:.2e}")
    assert err <= TOL["bf16"]


def test_sparse_full_selection_equals_dense():
    lens, n_q = (130, 67, 200), 2
    w, host, prob = _problem(lens, n_q, max(lens), seed=7)
    sel = torch.zeros(len(lens), n_q, max(lens), dtype=torch.int32)
    n_sel = torch.zeros(len(lens), n_q, dtype=torch.int32)
    for b, L in enumerate(lens):
        for j in range(n_q):
            p = L - n_q + j
            sel[b, j, : p + 1] = torch.arange(p + 1, dtype=torch.int32)
            n_sel[b, j] = p + 1
    prob.sel.copy_(sel)
    prob.n_sel.copy_(n_sel)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    sparse_out = prob.out.clone()
    dense = DeviceProblem(w.with_(top_k=0), host)
    dense.step()
    torch.cuda.synchronize()
    assert dense.get_status() == 0
    s_np = sparse_out.double().cpu().numpy()
    d_np = dense.out.double().cpu().numpy()
    assert np.isfinite(s_np).all() and np.isfinite(d_np).all()
    assert rel_err(s_np, d_np) <= TOL["bf16"]
    k_rot = O.rope_cache(host["k_rope"], host["seq_lens"], w.rope_base)
    ref = O.decode_naive(host["q_nope"], host["q_rope"], host["W_uk"], host["W_uv"], host["c_kv"], k_rot,
                         host["seq_lens"], n_q, w.softmax_scale, w.rope_base)
    assert rel_err(s_np, ref) <= TOL["bf16"] and rel_err(d_np, ref) <= TOL["bf16"]


def test_sparse_bad_count_zeroes_the_query():
    w, host, prob = _problem((130, 67, 200), 1, 40, seed=9)
    n_sel = host["n_sel"].clone()
    n_sel[1, 0] = 0
    n_sel[2, 0] = 41                      # > max_sel
    prob.n_sel.copy_(n_sel)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == B.CODES["MLA_ERR_LEN"]
    out = prob.out.float().cpu()
    assert torch.count_nonzero(out[1:]) == 0
    ref = _oracle(w, host, host["sel"].numpy(), host["n_sel"].numpy(), heads=HEADS)
    assert rel_err(out[:1, :, HEADS].double().numpy(), ref[:1, :, HEADS]) <= TOL["bf16"]


def test_sparse_slot_past_the_query_is_reported():
    w, host, prob = _problem((130, 67), 1, 40, seed=10)
    sel = host["sel"].clone()
    sel[1, 0, 5] = 67                     # the query sits at position 66
    prob.sel.copy_(sel)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == B.CODES["MLA_ERR_INDEX"]
    assert torch.isfinite(prob.out.float()).all()
