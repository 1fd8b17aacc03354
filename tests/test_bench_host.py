"""Host logic of the bench and the input generator (no GPU).

* W_O is drawn after every other input, so a workload with the output
  projection has the same queries, cache and weights as the one without;
* the reference arm's head sample projects a subset of the heads: the
  projections of disjoint head subsets add up to the projection of all heads;
* the roofline counts the output projection's bytes: W_O once, the head
  outputs once, y once."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from mla_latent_kv_43_b200 import inputs as gen  # noqa: E402
from mla_latent_kv_43_b200 import roofline as RF  # noqa: E402
from oracle import mla_oracle as O  # noqa: E402


def test_w_o_draw_leaves_the_other_inputs_unchanged():
    w = gen.tiny("fp32", lens=(9, 13), n_q=2, seed=3)
    a, b = gen.generate(w), gen.generate(w.with_(hidden_out=11))
    assert set(b) - set(a) == {"W_O"} and b["W_O"].shape == (w.heads * w.v_dim, 11)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_head_subset_projections_add_up():
    w = gen.tiny("fp32", lens=(9, 13), n_q=2, seed=4, heads=4, hidden_out=6)
    host = gen.generate(w)
    full = bench.oracle_decode(O, w, host, [0, 1])
    halves = bench.oracle_decode(O, w, host, [0, 1], heads=[0, 2]) + \
        bench.oracle_decode(O, w, host, [0, 1], heads=[1, 3])
    assert full.shape == (w.batch * w.n_q, 6)
    np.testing.assert_allclose(halves, full, rtol=1e-12, atol=1e-12)
    # and the full projection is the decode output times W_O
    dec = O.decode_step(host, w.n_q, w.d_c, w.softmax_scale).reshape(w.batch * w.n_q, -1)
    np.testing.assert_allclose(full, dec @ host["W_O"].double().numpy(), rtol=1e-12, atol=1e-12)


def test_roofline_counts_the_output_projection():
    w = gen.WORKLOADS["v3_b64_ragged_oproj"]
    lens = [2048] * w.batch
    K = w.heads * w.v_dim
    expect = (K * w.hidden_out + 64 * K + 64 * w.hidden_out) * 2
    assert RF.kernel_bytes("sm100_oproj", w, lens, 2, 2) == expect
    base = RF.step_work(gen.WORKLOADS["v3_b64_ragged"], lens)
    got = RF.step_work(w, lens)
    assert got["bytes"] - base["bytes"] == expect
    assert got["flops"] - base["flops"] == 2 * 64 * K * w.hidden_out


def test_prefill_flop_counts():
    """Causal pairs in closed form equal the count by brute force; the
    prefill's kernels count the materialised factorisation's FLOPs."""
    w = gen.tiny("bf16", lens=(7, 12, 30), n_q=5, prefill=True, heads=3, d_c=8, d_rope=4, qk_nope=6, v_dim=5)
    lens = [7, 12, 30]
    brute = sum(1 for L in lens for j in range(w.n_q) for k in range(L) if k <= L - w.n_q + j)
    assert RF.visible_pairs(w, lens) == brute
    assert RF.kernel_flops("sm100_prefill_attend", w, lens) == 2 * 3 * (6 + 4 + 5) * brute
    assert RF.kernel_flops("sm100_prefill_expand", w, lens) == 2 * sum(lens) * 8 * 3 * (6 + 5)
    assert RF.kernel_bytes("sm100_prefill_attend", w, lens, 2, 2) == 0.0
    step = RF.step_work(w, lens)
    assert step["flops"] == RF.kernel_flops("sm100_prefill_attend", w, lens) + \
        RF.kernel_flops("sm100_prefill_expand", w, lens)


def test_crossover_workloads():
    """The crossover sweep's workloads: one 4096-token sequence whose last n_q
    tokens are queries; the absorbed form's FLOPs grow with n_q faster than the
    materialised form's, which pays the expansion once."""
    lens = [4096]
    f = {}
    for n in bench.CROSSOVER_NQ:
        w = bench.crossover_workload(n)
        assert w.batch == 1 and w.lens == (4096,) and w.n_q == n and not w.prefill
        f[n] = (RF.step_work(w, lens)["flops"], RF.step_work(w.with_(prefill=True), lens)["flops"])
    assert f[1][0] < f[1][1]            # one query: absorbing is cheaper
    assert f[4096][0] > f[4096][1]      # a whole prompt: materialising is cheaper


def test_generated_scores_have_unit_variance():
    """Scale sanity of the input recipe: with the drawn distributions the scaled
    score q.k / sqrt(qk_nope + d_rope) has variance 1 (latent rows of unit RMS
    or unit variance, W ~ N(0, 1/d_c), queries and rope keys ~ N(0, 1)), so a
    mis-scaled weight or a wrong scale shows up here.  RoPE preserves norms and
    is left out."""
    for w in (gen.WORKLOADS["tiny_fp32"],
              gen.tiny("fp32", lens=(600, 600), heads=4, d_c=512, d_rope=64, qk_nope=128, v_dim=128,
                       latent_rms_norm=True, seed=9)):
        host = gen.generate(w)
        c = host["c_kv"].double().numpy()          # [B][cap][d_c]
        kr = host["k_rope"].double().numpy()
        qn = host["q_nope"].double().numpy()       # [B][n_q][H][qk_nope]
        qr = host["q_rope"].double().numpy()
        Wuk = host["W_uk"].double().numpy()        # [H][d_c][qk_nope]
        s = []
        for h in range(w.heads):
            K = c @ Wuk[h]                         # [B][cap][qk_nope]
            sc = (np.einsum("bk,bnk->bn", qn[:, 0, h], K) + np.einsum("bk,bnk->bn", qr[:, 0, h], kr))
            s.append(sc.ravel() * w.softmax_scale)
        std = float(np.std(np.concatenate(s)))
        assert 0.85 < std < 1.15, (w.name, std)


def test_step_work_matches_hand_counts():
    """Per-step algorithmic bytes and FLOPs of the DeepSeek-V3 workloads,
    counted by hand from the shapes: 1152 B per cached key read once per
    sequence, W_uk + W_uv = 33.55 MB, 49,152 B of queries and 32,768 B of
    outputs per query token, 278,528 FLOPs per visible (query, key) pair and
    33.55 MFLOPs of projections per query token (+ W_dkv, x and the new rows
    and 2 * 64 * 7168 * 576 FLOPs for the two appended tokens of 32
    sequences)."""
    W, QO, PAIR, PROJ = 33_554_432, 49_152 + 32_768, 278_528, 33_554_432
    cases = {
        "v3_b1_ctx8192": ([8192], 8192 * 1152 + W + QO, 8192 * PAIR + PROJ),
        "v3_b4_ctx131072": ([131072] * 4, 4 * 131072 * 1152 + W + 4 * QO, 4 * 131072 * PAIR + 4 * PROJ),
        # two causal queries per sequence see 4097 and 4098 keys
        "v3_b32_append2": ([4098] * 32,
                           32 * 4098 * 1152 + W + 7168 * 576 * 2 + 64 * 7168 * 2 + 64 * 576 * 2 + 64 * QO,
                           32 * (4097 + 4098) * PAIR + 64 * PROJ + 2 * 64 * 7168 * 576),
    }
    for name, (lens, nbytes, flops) in cases.items():
        r = RF.step_work(gen.WORKLOADS[name], lens)
        assert r["bytes"] == nbytes, (name, r["bytes"], nbytes)
        assert r["flops"] == flops, (name, r["flops"], flops)
    # the rounded figures: 43.07 MB / 2.32 GFLOP, 637.9 MB / 146.2 GFLOP, 199.1 MB / 75.7 GFLOP
    assert round(cases["v3_b1_ctx8192"][1] / 1e4) == 4307 and round(cases["v3_b32_append2"][2] / 1e8) == 757
    assert RF.cache_bytes_per_token(512, 64, 2) == 1152
    assert RF.cache_bytes_per_token(512, 64, 2, layers=61) == 70272


def test_attention_roofline_counts_cache_rows_only():
    """The attention kernel's algorithmic bytes are the cache rows (1152 B per
    key of each sequence); its absorbed queries and weighted latents are
    workspace intermediates, reported separately."""
    w = gen.WORKLOADS["v3_b64_ragged"]
    lens = [1000, 2048, 4096]
    assert RF.kernel_bytes("sm100_attend", w, lens, 2, 2) == sum(lens) * 1152
    assert RF.kernel_intermediate_bytes("sm100_attend", w, 2, 2) == w.batch * 128 * (576 + 512) * 2
    assert RF.kernel_intermediate_bytes("sm100_upproj", w, 2, 2) == 0.0
