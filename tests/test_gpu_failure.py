"""Failure detection without a GPU fault, and guard bytes around the outputs.

* The bounded wait every kernel uses gives up, records MLA_ERR_TIMEOUT and
  leaves normally: a wait on a barrier nothing arrives on (self-test entry
  point) reports the status, and the same context then decodes correctly.
* Decode writes nothing outside its output and workspace: guard bytes in
  front of and behind both keep their pattern (CUDA-core and tensor-core
  paths)."""
import os
import sys
import time

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


def _decode_check(w, host, prob, heads):
    prob.step()
    torch.cuda.synchronize()
    assert prob.get_status() == 0
    ref = O.decode_step(host, w.n_q, w.d_c, w.softmax_scale, heads=heads)
    got = prob.out.double().cpu().numpy()
    assert rel_err(got[:, :, heads], ref[:, :, heads]) <= TOL[w.dtype]


def test_bounded_wait_times_out_and_the_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    B.mla_selftest_wait_timeout(status, 50_000_000)          # 50 ms
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert B.mla_get_status(status) == B.CODES["MLA_ERR_TIMEOUT"]
    assert 0.04 < dt < 5.0, dt
    # the context is intact: a decode on the tensor-core path still matches the oracle
    w = gen.tiny("bf16", lens=(130, 67), seed=21, latent_rms_norm=True, **V3)
    host = gen.generate(w)
    _decode_check(w, host, DeviceProblem(w, host), heads=[0, 64, 127])


@pytest.mark.parametrize("geom", ["fp32_small", "bf16_v3"])
def test_decode_writes_nothing_outside_its_buffers(geom):
    if geom == "fp32_small":
        w = gen.tiny("fp32", lens=(7, 40, 129), n_q=2, seed=22, heads=3, d_c=8, d_rope=4, qk_nope=6, v_dim=5)
    else:
        w = gen.tiny("bf16", lens=(130, 67, 200), n_q=2, seed=22, latent_rms_norm=True, **V3)
    host = gen.generate(w)
    prob = DeviceProblem(w, host)
    G = 4096                                                 # guard bytes on each side (16-byte multiple)
    pattern = 0xA5
    # output: the same shape, carved out of a larger byte buffer
    out_bytes = prob.out.numel() * prob.out.element_size()
    obuf = torch.full((G + out_bytes + G,), pattern, dtype=torch.uint8, device="cuda")
    prob.out = obuf[G: G + out_bytes].view(prob.out.dtype).view(prob.out.shape)
    ws_bytes = prob.workspace.numel()
    wbuf = torch.full((G + ws_bytes + G,), pattern, dtype=torch.uint8, device="cuda")
    prob.workspace = wbuf[G: G + ws_bytes]
    heads = [0, w.heads - 1]
    _decode_check(w, host, prob, heads)
    for buf, n in ((obuf, out_bytes), (wbuf, ws_bytes)):
        head, tail = buf[:G].cpu().numpy(), buf[G + n:].cpu().numpy()
        assert (head == pattern).all() and (tail == pattern).all()
