"""Drive libmla on one GPU for a generated workload.

A ``DeviceProblem`` holds a workload's tensors on the device, in the layout
the library takes: the cache as [B][capacity][d_c + d_rope] with its rope
keys rotated at their slot positions by ``mla_rope`` (what the append step
would have stored), the weights, per-sequence lengths, and caller-owned
output, workspace and status buffers.  ``step()`` runs one decode step
(append of the new tokens when the workload has them, then attention: over
every visible key, or over the selected ones for a top-k workload; in the
materialised factorisation for a prefill workload), then,
when the workload has a W_O, the output projection into ``y``.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import binding as B
from .inputs import Workload


class DeviceProblem:
    def __init__(self, w: Workload, host: Dict[str, torch.Tensor], device="cuda", splits: int = 0,
                 stream: Optional[torch.cuda.Stream] = None, max_len: Optional[int] = None):
        self.w = w
        self.dims = B.dims_of(w)
        self.splits = splits
        self.stream = stream
        dev = torch.device(device)
        self.device = dev
        to = lambda t: t.to(dev, non_blocking=False).contiguous()
        self.q_nope = to(host["q_nope"])
        self.q_rope = to(host["q_rope"])
        self.W_uk = to(host["W_uk"])
        self.W_uv = to(host["W_uv"])
        self.seq_lens = to(host["seq_lens"])
        self.max_len = int(host["seq_lens"].max()) if max_len is None else int(max_len)
        # cache = [latent || raw rope key] per slot, then rotate every slot's rope
        # key at its position inside the sequence.
        self.cache = torch.empty(w.batch, w.capacity, w.d, dtype=w.torch_dtype, device=dev)
        self.cache[..., : w.d_c].copy_(host["c_kv"])
        self.cache[..., w.d_c:].copy_(host["k_rope"])
        slot_pos = torch.arange(w.capacity, dtype=torch.int32, device=dev).repeat(w.batch)
        B.mla_rope(self.dims, w.batch * w.capacity, self.cache, w.d, slot_pos, stream=stream,
                   offset_elems=w.d_c)
        del slot_pos
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.out = torch.empty(w.batch, w.n_q, w.heads, w.v_dim, dtype=w.torch_dtype, device=dev)
        self.sparse = w.top_k > 0
        if self.sparse:
            self.sel = to(host["sel"])
            self.n_sel = to(host["n_sel"])
        self.prefill = w.prefill
        ws_len = w.top_k if self.sparse else self.max_len    # the tile bound of the plan
        if self.prefill:
            self.layout = {"total": B.mla_prefill_workspace_bytes(self.dims, w.batch, w.n_q, self.max_len)}
        else:
            self.layout = B.mla_decode_workspace_layout(self.dims, w.batch, w.n_q, ws_len, splits)
        self.workspace = torch.empty(max(self.layout["total"], 256), dtype=torch.uint8, device=dev)
        self.has_oproj = w.hidden_out > 0
        if self.has_oproj:
            self.W_O = to(host["W_O"])
            self.y = torch.empty(w.batch * w.n_q, w.hidden_out, dtype=w.torch_dtype, device=dev)
        self.has_append = w.n_new > 0
        if self.has_append:
            self.x = to(host["x"])
            self.W_dkv = to(host["W_dkv"])
            self.positions = to(host["positions"])

    # --- the step -----------------------------------------------------------
    def append(self):
        B.mla_append(self.dims, self.x, self.W_dkv, self.positions, self.cache, self.status,
                     batch=self.w.batch, n_new=self.w.n_new, stream=self.stream)

    def decode(self):
        if self.prefill:
            B.mla_prefill(self.dims, self.q_nope, self.q_rope, self.W_uk, self.W_uv, self.cache, self.seq_lens,
                          self.max_len, self.out, self.workspace, self.status, stream=self.stream)
            return
        if self.sparse:
            B.mla_decode_sparse(self.dims, self.q_nope, self.q_rope, self.W_uk, self.W_uv, self.cache,
                                self.seq_lens, self.max_len, self.sel, self.n_sel, self.out, self.workspace,
                                self.status, splits=self.splits, stream=self.stream)
            return
        B.mla_decode(self.dims, self.q_nope, self.q_rope, self.W_uk, self.W_uv, self.cache,
                     self.seq_lens, self.max_len, self.out, self.workspace, self.status,
                     splits=self.splits, stream=self.stream)

    def project(self):
        B.mla_output_projection(self.dims, self.out, self.W_O, self.y, self.status, stream=self.stream)

    def step(self) -> int:
        """One decode step; returns the number of kernels it enqueued."""
        n = 0
        if self.has_append:
            self.append()
            n += B.mla_last_launch_count()
        self.decode()
        n += B.mla_last_launch_count()
        if self.has_oproj:
            self.project()
            n += B.mla_last_launch_count()
        return n

    @property
    def result(self) -> torch.Tensor:
        """What the step hands back: y after the output projection, else the head outputs."""
        return self.y if self.has_oproj else self.out

    def get_status(self) -> int:
        return B.mla_get_status(self.status, stream=self.stream)

    def workspace_view(self, region: str, shape, dtype) -> torch.Tensor:
        off, nbytes = self.layout[region], self.layout[region + "_bytes"]
        t = self.workspace[off: off + nbytes].view(dtype)
        return t.view(*shape)
