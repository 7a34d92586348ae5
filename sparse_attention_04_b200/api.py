"""Convenience layer over the C ABI for torch users.

Allocates outputs and workspaces as torch CUDA tensors (PyTorch is used for
device memory and streams only) and calls the library through `_lib`.  Every
step of the path runs in the library's kernels.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import _lib
from .inputs import D_V, Inputs


@dataclasses.dataclass
class StepResult:
    out: torch.Tensor           # [B,T,H,512]
    lse: torch.Tensor           # [B,T,H] fp32
    scores: torch.Tensor        # [B*T, ld] fp32 (a view of the workspace for decode)
    indices: torch.Tensor       # [B*T, k] int32
    status: torch.Tensor        # int32 [1], device
    ld: int


def _out_dtype(wl):
    return torch.float32 if wl.out_dtype == "f32" else torch.bfloat16


class DecodeStep:
    """Buffers for repeated dsa_decode_step calls on one workload shape."""

    def __init__(self, B: int, max_end_pos: int, k: int, H: int, out_dtype=torch.bfloat16, device="cuda"):
        self.B, self.max_end_pos, self.k, self.H = B, max_end_pos, k, H
        nbytes = _lib.decode_step_workspace_size(B, max_end_pos, k, H)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        so, ld, io, _ = _lib.decode_step_workspace_layout(B, max_end_pos, k, H)
        self.ld = ld
        self.scores = self.workspace[so:so + B * ld * 4].view(torch.float32).view(B, ld)
        self.indices = self.workspace[io:io + B * k * 4].view(torch.int32).view(B, k)
        self.out = torch.empty((B, 1, H, D_V), dtype=out_dtype, device=device)
        self.lse = torch.empty((B, 1, H), dtype=torch.float32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, q_idx, w, k_idx, k_scale, q, kv, offsets, kv_rows, scale, stream=None):
        _lib.decode_step(q_idx, w, k_idx, k_scale, q, kv, offsets, self.B, self.max_end_pos, kv_rows,
                         self.k, self.H, scale, self.out, lse=self.lse, workspace=self.workspace,
                         status=self.status, stream=stream)
        return self.out


def decode_step(inp: Inputs, step: Optional[DecodeStep] = None) -> StepResult:
    """Runs the fused decode step (T must be 1) on device-resident inputs."""
    wl = inp.wl
    assert wl.T == 1
    if step is None:
        step = DecodeStep(wl.B, max(inp.end_pos), wl.topk, wl.H, _out_dtype(wl), inp.q.device)
    step(inp.q_idx, inp.w, inp.k_idx, inp.k_scale, inp.q, inp.kv, inp.offsets, inp.rows, wl.scale)
    return StepResult(step.out, step.lse, step.scores, step.indices, step.status, step.ld)


def staged(inp: Inputs) -> StepResult:
    """Runs the three stages as separate calls (any T, e.g. causal prefill)."""
    wl = inp.wl
    dev = inp.q.device
    B, T, H, k = wl.B, wl.T, wl.H, wl.topk
    n = B * T
    ld = (max(inp.end_pos) + 3) // 4 * 4
    scores = torch.empty((n, ld), dtype=torch.float32, device=dev)
    indices = torch.empty((n, k), dtype=torch.int32, device=dev)
    out = torch.empty((B, T, H, D_V), dtype=_out_dtype(wl), device=dev)
    lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws_bytes = _lib.sparse_mla_workspace_size(B, T, H, k)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _lib.indexer_scores(inp.q_idx, inp.w, inp.k_idx, inp.k_scale, inp.offsets, B, T, inp.rows, scores, ld,
                        status=status)
    _lib.topk(scores, ld, inp.offsets, B, T, k, indices, status=status)
    _lib.sparse_mla(inp.q, inp.kv, inp.offsets, indices, B, T, H, k, wl.scale, inp.rows, out, lse=lse,
                    workspace=ws, status=status)
    return StepResult(out, lse, scores, indices, status, ld)
