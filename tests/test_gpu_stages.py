"""Intermediate results of one decode call against the oracle's absorbed
form: the absorbed queries q_lat = [W_uk q_nope || RoPE(q_rope)], the
softmax-weighted latents o_lat, and the final outputs -- so a failure points
at one kernel.  Runs both the CUDA-core geometry and the DeepSeek-V3
geometry (tensor-core path), with several split counts."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from gpu_common import TOL, gpu_out, rel_err  # noqa: E402
from mla_latent_kv_43_b200 import inputs as gen  # noqa: E402
from mla_latent_kv_43_b200.runner import DeviceProblem  # noqa: E402
from oracle import mla_oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu

SMALL = dict(heads=3, d_c=8, d_rope=4, qk_nope=6, v_dim=5)
V3 = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128)


def merge_pieces(prob, o_lat, BJ, H, d_c):
    """The tensor-core path leaves a query token whose key tiles were cut across
    work items as pieces (normalised partial rows, one log2-sum-exp per latent
    half); merge them here as the up-projection does after projecting.  Item p
    covers tiles [start[p], start[p + 1]) (from the schedule); a cut token's
    first piece is in slot 2 pf + 1, its later ones in slot 2 p."""
    P = prob.layout["splits"]
    sched = prob.workspace_view("sched", (-1,), torch.int32).cpu().numpy().astype(np.int64)
    cum = sched[: BJ + 1]
    start = list(sched[BJ + 1 + 3 * P: BJ + 2 + 4 * P])          # each item's first key tile
    # part_o head-major, blocked by 64 columns: [H][d_c / 64][2P][64]; part_lse [H][2P][2]
    part_o = prob.workspace_view("part_o", (H, d_c // 64, 2 * P, 64), torch.bfloat16).double().cpu().numpy()
    part_o = part_o.transpose(2, 0, 1, 3).reshape(2 * P, H, d_c)
    lse = prob.workspace_view("part_lse", (H, 2 * P, 2), torch.float32).double().cpu().numpy().transpose(1, 2, 0)
    pair_of = lambda t: max(p for p in range(P) if start[p] <= t)  # noqa: E731
    out = o_lat.copy()
    for n in range(BJ):
        c0, c1 = cum[n], cum[n + 1]
        if c1 == c0:
            continue
        pf, pl = pair_of(c0), pair_of(c1 - 1)
        if pf == pl:
            continue
        slots = [2 * pf + 1] + [2 * p for p in range(pf + 1, pl + 1) if start[p] < start[p + 1]]
        half = d_c // 2
        for r in range(2):
            lw = lse[slots, r, :]                                   # [pieces][H]
            wts = np.exp2(lw - lw.max(axis=0))
            wts /= wts.sum(axis=0)
            out[n, :, r * half:(r + 1) * half] = np.einsum("ph,phc->hc", wts,
                                                           part_o[slots][:, :, r * half:(r + 1) * half])
    return out


def run_and_compare(dtype, g, lens, n_q, splits, heads):
    w = gen.tiny(dtype, lens=lens, n_q=n_q, seed=11, latent_rms_norm=(g is V3), **g)
    host = gen.generate(w)
    prob = DeviceProblem(w, host, splits=splits)
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    L = prob.layout
    cdt = torch.bfloat16 if L["compute_dtype"] == 0 else torch.float32
    BJ = w.batch * n_q
    q_lat = prob.workspace_view("q_lat", (BJ, w.heads, w.d), cdt).double().cpu().numpy()
    o_lat = prob.workspace_view("o_lat", (BJ, w.heads, w.d_c), cdt).double().cpu().numpy()
    if L["compute_dtype"] == 0:
        o_lat = merge_pieces(prob, o_lat, BJ, w.heads, w.d_c)
    out = gpu_out(prob)
    k_rot = O.rope_cache(host["k_rope"], host["seq_lens"])
    ref_out, inter = O.decode_absorbed(host["q_nope"], host["q_rope"], host["W_uk"], host["W_uv"],
                                       host["c_kv"], k_rot, host["seq_lens"], n_q, w.softmax_scale,
                                       heads=heads, return_intermediates=True)
    keys = sorted(inter)
    g_q = np.stack([q_lat[b * n_q + j, h] for b, j, h in keys])
    r_q = np.stack([inter[k][0] for k in keys])
    g_o = np.stack([o_lat[b * n_q + j, h] for b, j, h in keys])
    r_o = np.stack([inter[k][1] for k in keys])
    g_y = np.stack([out[b, j, h] for b, j, h in keys])
    r_y = np.stack([ref_out[b, j, h] for b, j, h in keys])
    errs = (rel_err(g_q, r_q), rel_err(g_o, r_o), rel_err(g_y, r_y))
    print(f"{dtype} H={w.heads} lens={lens} n_q={n_q} splits={splits}: "
          f"q_lat {errs[0]:.2e}  o_lat {errs[1]:.2e}  out {errs[2]:.2e}")
    tol = TOL[dtype]
    assert errs[0] <= tol, ("q_lat", errs)
    assert errs[1] <= tol, ("o_lat", errs)
    assert errs[2] <= tol, ("out", errs)


@pytest.mark.parametrize("n_q", [1, 2])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_v3_stages(n_q, splits):
    run_and_compare("bf16", V3, (130, 67, 200), n_q, splits, heads=[0, 1, 31, 32, 63, 64, 95, 96, 127])


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_small_stages(dtype):
    run_and_compare(dtype, SMALL, (7, 40, 129), 2, 0, heads=None)
