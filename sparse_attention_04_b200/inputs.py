"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) decode/prefill path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no scores, no selection, no attention).  Both the CUDA
path and the fp64 oracle are fed the exact same bytes produced here.

Workloads (shapes follow the DeepSeek-V3.2-Exp indexer and MLA tensors as the
pages print them: "DeepSeek-V3.2-Exp - Keep top-k positions", Indexer.forward;
"DeepSeek-V3.2-Exp - Apply sparse mask", MQA decode branch):

  tiny       B=1,  T=1,    end_pos=256,             topk=64,   H=16,  bf16 indexer
  decode32k  B=1,  T=1,    end_pos=32768,           topk=2048, H=128, bf16 indexer
  batched    B=32, T=1,    end_pos ~ U[8192,131072], topk=2048, H=128, bf16 indexer
  prefill4k  B=1,  T=4096, end_pos=4096 (causal),    topk=2048, H=128, bf16 indexer
  fp8        B=4,  T=1,    end_pos=131072,          topk=2048, H=128, e4m3 indexer
  decode2k   B=1,  T=1,    end_pos=2048,            topk=2048, H=128, bf16 indexer
             (short context: every position kept, indexer and selection skipped)

Draw recipe (one torch.Generator seeded with the workload's seed, on the
device the tensors are made on, draws taken in this order):
  1. end_pos per sequence (batched only): integers uniform in [8192, 131072]
  2. q_idx [B,T,64,128] ~ N(0,1), rounded to bf16 (round-to-nearest-even)
  3. w     [B,T,64]      ~ N(0,1) * 64^-0.5 * 128^-0.5, fp32
  4. k_idx [rows,128]    ~ N(0,1), bf16
  5. q     [B,T,H,576]   ~ N(0,1), bf16  (absorbed latent query: 512 latent + 64 rope)
  6. kv    [rows,576]    ~ N(0,1), bf16  (512 latent || 64 rope per cached token)
For the e4m3 workload, q_idx and k_idx (already bf16) are quantised per
128-element block (one block per head vector / per key, since the indexer head
dim is 128) with scale = amax/448 and a round-to-nearest-even cast to e4m3;
the q scale is folded into w, as the Indexer.forward listing does before it
calls fp8_index.  This quantisation is input synthesis: the cache the kernels
read is already e4m3, exactly like the reference's k_cache.

Caches are stored ragged: sequence b owns rows [offsets[b], offsets[b+1]) of
both the indexer key cache and the latent cache; end_pos_b = offsets[b+1]-offsets[b].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

H_I = 64      # indexer heads (index_n_heads)
D_I = 128     # indexer head dim (index_head_dim)
D_QK = 576    # latent (512) + rope (64)
D_V = 512     # latent width used as V
E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    end_pos: Optional[int]          # fixed end_pos for every sequence, or None (drawn)
    end_pos_range: Optional[tuple]  # inclusive [lo, hi] when drawn
    topk: int
    H: int
    idx_dtype: str                  # "bf16" | "e4m3"
    scale: float                    # MLA softmax scale
    out_dtype: str                  # "f32" | "bf16"
    seed: int


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 256, None, 64, 16, "bf16", 576 ** -0.5, "f32", 0),
    "decode32k": Workload("decode32k", 1, 1, 32768, None, 2048, 128, "bf16", 192 ** -0.5, "bf16", 1),
    "batched": Workload("batched", 32, 1, None, (8192, 131072), 2048, 128, "bf16", 192 ** -0.5, "bf16", 2),
    "prefill4k": Workload("prefill4k", 1, 4096, 4096, None, 2048, 128, "bf16", 192 ** -0.5, "bf16", 3),
    "fp8": Workload("fp8", 4, 1, 131072, None, 2048, 128, "e4m3", 192 ** -0.5, "bf16", 4),
    # short context: end_pos <= topk, so every position is kept and the decode
    # step skips the indexer and the selection
    "decode2k": Workload("decode2k", 1, 1, 2048, None, 2048, 128, "bf16", 192 ** -0.5, "bf16", 5),
}


def custom(name="custom", B=1, T=1, end_pos=256, topk=64, H=16, idx_dtype="bf16",
           scale=None, out_dtype="f32", seed=0, end_pos_range=None) -> Workload:
    """A workload with the same distributions and arbitrary sizes (tests use it)."""
    if scale is None:
        scale = D_QK ** -0.5
    return Workload(name, B, T, end_pos, end_pos_range, topk, H, idx_dtype, scale, out_dtype, seed)


@dataclasses.dataclass
class Inputs:
    wl: Workload
    end_pos: list            # python ints, per sequence
    offsets: torch.Tensor    # int32 [B+1]
    q_idx: torch.Tensor      # bf16 [B,T,64,128] or uint8 (e4m3 bytes) [B,T,64,128]
    w: torch.Tensor          # fp32 [B,T,64] (q scale folded in for e4m3)
    k_idx: torch.Tensor      # bf16 [rows,128] or uint8 (e4m3 bytes) [rows,128]
    k_scale: Optional[torch.Tensor]  # fp32 [rows] for e4m3, else None
    q: torch.Tensor          # bf16 [B,T,H,576]
    kv: torch.Tensor         # bf16 [rows,576]

    @property
    def rows(self) -> int:
        return int(sum(self.end_pos))

    def to(self, device) -> "Inputs":
        mv = lambda t: None if t is None else t.to(device)
        return Inputs(self.wl, list(self.end_pos), mv(self.offsets), mv(self.q_idx), mv(self.w),
                      mv(self.k_idx), mv(self.k_scale), mv(self.q), mv(self.kv))


def _randn_bf16(gen, shape, device, chunk=1 << 26):
    """N(0,1) drawn in fp32 and rounded to bf16 (torch's cast is round-to-nearest-even)."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        out[lo:hi] = torch.randn(hi - lo, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def quantize_e4m3_blocks(x: torch.Tensor):
    """Per-row (128-element block) e4m3 quantisation of a [..., 128] tensor.

    Returns (uint8 codes with the same leading shape, fp32 scales [...]).
    scale = amax / 448 (amax == 0 -> scale 1), value = x / scale cast to e4m3 (RNE).
    """
    assert x.shape[-1] == D_I
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (xf / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.float()


def make_inputs(wl: Workload, device="cpu", end_pos: Optional[Sequence[int]] = None) -> Inputs:
    """Draw the workload's inputs on `device` with the documented recipe."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    B, T, H = wl.B, wl.T, wl.H
    if end_pos is not None:
        ep = [int(e) for e in end_pos]
        assert len(ep) == B
    elif wl.end_pos is not None:
        ep = [int(wl.end_pos)] * B
    else:
        lo, hi = wl.end_pos_range
        ep = torch.randint(lo, hi + 1, (B,), generator=gen, device=device).tolist()
    assert all(e >= T for e in ep), "end_pos must cover the T query rows"
    offs = [0]
    for e in ep:
        offs.append(offs[-1] + e)
    rows = offs[-1]
    offsets = torch.tensor(offs, dtype=torch.int32, device=device)

    q_idx = _randn_bf16(gen, (B, T, H_I, D_I), device)
    w = torch.randn((B, T, H_I), generator=gen, device=device, dtype=torch.float32) * (H_I ** -0.5) * (D_I ** -0.5)
    k_idx = _randn_bf16(gen, (rows, D_I), device)
    q = _randn_bf16(gen, (B, T, H, D_QK), device)
    kv = _randn_bf16(gen, (rows, D_QK), device)
    k_scale = None
    if wl.idx_dtype == "e4m3":
        q_idx, q_scale = quantize_e4m3_blocks(q_idx)
        w = (w * q_scale).float()
        k_idx, k_scale = quantize_e4m3_blocks(k_idx)
    elif wl.idx_dtype != "bf16":
        raise ValueError(wl.idx_dtype)
    return Inputs(wl, ep, offsets, q_idx.contiguous(), w.contiguous(), k_idx.contiguous(),
                  k_scale, q.contiguous(), kv.contiguous())
