"""Convenience layer over the C ABI for torch users.

Allocates outputs and workspaces as torch CUDA tensors (PyTorch is used for
device memory and streams only) and calls the library through `_lib`.  Every
step of the path runs in the library's kernels.
"""
from __future__ import annotations

import dataclasses
import math
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


class HostDecodeStep:
    """A decode step fed from pinned host memory whose output goes back to
    pinned host memory: the form a server uses when the new token's
    projections arrive from the host.

    The caller fills the pinned views host_q_idx [B,1,64,128] bf16, host_w
    [B,1,64] fp32, host_k_new [B,1,128] bf16, host_kv_new [B,1,576] bf16 and
    host_q [B,1,H,576] bf16, calls the object with the resident caches, and
    reads host_out [B,1,H,512] once the stream has been synchronised (and only
    then refills the inputs).  One call issues on the current stream

        copy kernel (q_I, w, k_new, kv_new) -> dsa_cache_append
        -> [dsa_quantize_queries for e4m3 keys] -> dsa_indexer_scores
        -> dsa_topk -> dsa_sparse_mla -> copy kernel (out)

    How q, the largest input, crosses PCIe depends on its size (measured on
    B200, microseconds per host-fed step):
      - up to Q_WITH_INPUTS_MAX bytes (one 128-head row): in the same copy
        kernel as the small inputs, so that the whole dsa_decode_step follows
        with q complete and the attention loads its query tile before the
        selection ends (decode 32K: 36.3 against 37.5 with the side stream);
      - up to Q_KERNEL_COPY_MAX bytes: on a side stream, by a copy kernel
        launched once the indexer has finished, so it crosses PCIe while the
        selection runs on a few SMs; the attention waits for it.  Started with
        the step, its CTAs took registers that the indexer's CTAs needed and
        held them back (fp8 B=4: 78.8 against 71.4; in the first copy 78.1);
      - above that: by the copy engine on the side stream from the start of
        the step, so that a long transfer overlaps the indexer too and holds
        no SM.
    When every end_pos <= k the attention-only form of dsa_decode_step runs
    once q is in.  Each call starts after everything issued before it on the
    stream."""

    Q_WITH_INPUTS_MAX = 1 << 18
    Q_KERNEL_COPY_MAX = 1 << 20

    def __init__(self, B: int, max_end_pos: int, k: int, H: int, idx_dtype: str = "bf16",
                 out_dtype=torch.bfloat16, device="cuda"):
        dev = torch.device(device)
        self.step = DecodeStep(B, max_end_pos, k, H, out_dtype, dev)
        self.B, self.max_end_pos, self.k, self.H = B, max_end_pos, k, H
        self.fp8 = idx_dtype == "e4m3"
        # one pinned staging buffer for the small inputs (and q, when it is
        # small enough to travel with them), 256-byte aligned sections
        q_bytes = B * H * 576 * 2
        self.q_with_inputs = q_bytes <= self.Q_WITH_INPUTS_MAX
        spec = [(torch.bfloat16, (B, 1, 64, 128)), (torch.float32, (B, 1, 64)),
                (torch.bfloat16, (B, 1, 128)), (torch.bfloat16, (B, 1, 576))]
        if self.q_with_inputs:
            spec.append((torch.bfloat16, (B, 1, H, 576)))
        sizes = [math.prod(shape) * torch.empty((), dtype=dt).element_size() for dt, shape in spec]
        offs, tot = [], 0
        for sz in sizes:
            offs.append(tot)
            tot += -(-sz // 256) * 256
        self.host_small = torch.zeros(tot, dtype=torch.uint8, pin_memory=True)
        self._small = torch.empty(tot, dtype=torch.uint8, device=dev)

        def views(buf):
            return [buf[o:o + n].view(dt).view(*shape) for o, n, (dt, shape) in zip(offs, sizes, spec)]

        hv, dv = views(self.host_small), views(self._small)
        self.host_q_idx, self.host_w, self.host_k_new, self.host_kv_new = hv[:4]
        self._q_idx, self._w, self._k_new, self._kv_new = dv[:4]
        if self.q_with_inputs:
            self.host_q, self._q = hv[4], dv[4]
        else:
            self.host_q = torch.zeros((B, 1, H, 576), dtype=torch.bfloat16, pin_memory=True)
            self._q = torch.empty((B, 1, H, 576), dtype=torch.bfloat16, device=dev)
        self.host_out = torch.zeros(tuple(self.step.out.shape), dtype=out_dtype, pin_memory=True)
        if self.fp8:
            self._q8 = torch.empty((B, 1, 64, 128), dtype=torch.uint8, device=dev)
            self._w8 = torch.empty((B, 1, 64), dtype=torch.float32, device=dev)
        m_off = _lib.decode_step_workspace_layout(B, max_end_pos, k, H)[3]
        self._ws_mla = self.step.workspace[m_off:]
        self._side = torch.cuda.Stream(dev)
        self.h2d_bytes = tot + (0 if self.q_with_inputs else self.host_q.numel() * 2)
        self.d2h_bytes = self.host_out.numel() * self.host_out.element_size()

    def _copy_q(self, cur):
        """q's transfer on the side stream, after everything issued so far on `cur`."""
        self._side.wait_stream(cur)
        with torch.cuda.stream(self._side):
            if self.host_q.numel() * 2 <= self.Q_KERNEL_COPY_MAX:
                _lib.copy_host_to_device(self._q, self.host_q)
            else:
                self._q.copy_(self.host_q, non_blocking=True)

    def __call__(self, k_idx, k_scale, kv, offsets, kv_rows, scale):
        st, B = self.step, self.B
        cur = torch.cuda.current_stream()
        q_by_kernel = self.host_q.numel() * 2 <= self.Q_KERNEL_COPY_MAX
        short = self.max_end_pos <= self.k
        if not self.q_with_inputs and (short or not q_by_kernel):
            self._copy_q(cur)
        _lib.copy_host_to_device(self._small, self.host_small)
        _lib.cache_append(self._k_new, self._kv_new, offsets, B, 1, k_idx, k_scale, kv, kv_rows, status=st.status)
        q_idx, w = self._q_idx, self._w
        if self.fp8:
            _lib.quantize_queries(q_idx, w, B, self._q8, self._w8)
            q_idx, w = self._q8, self._w8
        if self.q_with_inputs:
            # q is complete before the step's first kernel: the fused step
            st(q_idx, w, k_idx, k_scale, self._q, kv, offsets, kv_rows, scale)
        elif short:
            cur.wait_stream(self._side)
            st(q_idx, w, k_idx, k_scale, self._q, kv, offsets, kv_rows, scale)
        else:
            _lib.indexer_scores(q_idx, w, k_idx, k_scale, offsets, B, 1, kv_rows, st.scores, st.ld,
                                status=st.status)
            if q_by_kernel:
                self._copy_q(cur)  # crosses PCIe beside the selection
            _lib.topk(st.scores, st.ld, offsets, B, 1, self.k, st.indices, status=st.status)
            cur.wait_stream(self._side)
            _lib.sparse_mla(self._q, kv, offsets, st.indices, B, 1, self.H, self.k, scale, kv_rows, st.out,
                            lse=st.lse, workspace=self._ws_mla, status=st.status)
        _lib.copy_device_to_host(self.host_out, st.out)
        return self.host_out


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
