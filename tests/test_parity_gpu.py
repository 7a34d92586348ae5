"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances (fixed by the task's correctness criteria):
  indexer scores   |gpu - ref| <= 1e-3 * (1 + |ref|), masked entries exactly -inf
  top-k indices    bit-exact to the oracle's selection run on the GPU's own
                   scores; >= 99.9 % set overlap with the selection on the
                   oracle's scores
  attention        |gpu - ref| <= 1e-2 + 1e-2 * |ref| (out and lse), with the
                   oracle run on the GPU's indices
Small cases are checked element by element in full; the full-size workloads
run in the same launch configuration the benchmark times and are checked on
sampled rows.
"""
import math

import pytest
import torch

import oracle
from sparse_attention_04_b200 import inputs as dsa_inputs
from sparse_attention_04_b200.inputs import Inputs

pytestmark = pytest.mark.gpu


def _api():
    from sparse_attention_04_b200 import api
    return api


# ------------------------------------------------------------------ helpers

def subset(inp: Inputs, seqs):
    """CPU copy of the inputs restricted to the listed sequences (rows renumbered)."""
    T = inp.wl.T
    off = inp.offsets.cpu().tolist()
    eps = [inp.end_pos[b] for b in seqs]
    new_off = [0]
    for e in eps:
        new_off.append(new_off[-1] + e)
    cat = lambda t: torch.cat([t[off[b]:off[b + 1]].cpu() for b in seqs])
    sel = lambda t: t[list(seqs)].cpu()
    wl = dsa_inputs.Workload(inp.wl.name, len(seqs), T, None, None, inp.wl.topk, inp.wl.H, inp.wl.idx_dtype,
                             inp.wl.scale, inp.wl.out_dtype, inp.wl.seed)
    return Inputs(wl, eps, torch.tensor(new_off, dtype=torch.int32), sel(inp.q_idx), sel(inp.w), cat(inp.k_idx),
                  None if inp.k_scale is None else cat(inp.k_scale), sel(inp.q), cat(inp.kv))


def check_scores(gpu, ref, E_of_row):
    gpu = gpu.double().cpu()
    for i, E in enumerate(E_of_row):
        g, r = gpu[i, :E], ref[i, :E]
        masked = torch.isinf(r)
        assert torch.all(torch.isinf(g[masked]) & (g[masked] < 0)), f"row {i}: masked entries"
        err = (g[~masked] - r[~masked]).abs()
        tol = 1e-3 * (1 + r[~masked].abs())
        assert torch.all(err <= tol), f"row {i}: max err {float(err.max())}"


def check_topk(gpu_idx, gpu_scores_rows, ref_scores_rows, sub: Inputs, rows):
    B, T, k = sub.wl.B, sub.wl.T, sub.wl.topk
    own = oracle.topk(gpu_scores_rows.double(), sub.offsets, B, T, k, rows=rows)
    assert torch.equal(gpu_idx.cpu(), own), "top-k differs from the oracle's selection on the GPU scores"
    ref = oracle.topk(ref_scores_rows, sub.offsets, B, T, k, rows=rows)
    inter = total = 0
    for a, b in zip(gpu_idx.cpu().tolist(), ref.tolist()):
        sa, sb = {x for x in a if x >= 0}, {x for x in b if x >= 0}
        inter += len(sa & sb)
        total += len(sb)
    assert inter >= 0.999 * total, f"overlap {inter}/{total}"


def check_mla(gpu_out, gpu_lse, gpu_idx, sub: Inputs, rows):
    wl = sub.wl
    ref, ref_lse = oracle.sparse_mla(sub.q, sub.kv, sub.offsets, gpu_idx.cpu(), wl.B, wl.T, wl.H, wl.topk,
                                     wl.scale, rows=rows)
    g = gpu_out.double().cpu()
    err = (g - ref).abs()
    assert torch.all(err <= 1e-2 + 1e-2 * ref.abs()), f"out max err {float(err.max())}"
    gl = gpu_lse.double().cpu()
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isfinite(gl), fin)
    assert torch.all((gl[fin] - ref_lse[fin]).abs() <= 1e-2 + 1e-2 * ref_lse[fin].abs())


def run_and_check(wl, device, rows=None, seqs=None, end_pos=None, staged=False, mutate=None):
    api = _api()
    inp = dsa_inputs.make_inputs(wl, device, end_pos=end_pos)
    if mutate:
        mutate(inp)
    # a decode step whose every end_pos <= k skips the indexer and the selection
    # (nothing to compare there): the stages are then checked one by one and
    # the fused step's dense output separately below
    short = wl.T == 1 and max(inp.end_pos) <= wl.topk
    res = api.staged(inp) if (staged or wl.T > 1 or short) else api.decode_step(inp)
    torch.cuda.synchronize()
    assert int(res.status.item()) == 0, _lib_status(res.status)
    seqs = list(range(wl.B)) if seqs is None else seqs
    sub = subset(inp, seqs)
    T = wl.T
    if rows is None:
        rows = list(range(len(seqs) * T))
    glob_rows = [seqs[r // T] * T + r % T for r in rows]
    E_of_row = [sub.end_pos[r // T] for r in rows]
    ld = max(sub.end_pos)
    ref = oracle.indexer_scores(sub.q_idx, sub.w, sub.k_idx, sub.k_scale, sub.offsets, sub.wl.B, T, ld, rows=rows)
    gpu_sc = res.scores[glob_rows][:, :ld].cpu()
    check_scores(gpu_sc, ref, E_of_row)
    gsc = torch.where(torch.arange(ld)[None, :] < torch.tensor(E_of_row)[:, None], gpu_sc.double(),
                      torch.tensor(float("nan"), dtype=torch.float64))
    gidx = res.indices[glob_rows].cpu()
    check_topk(gidx, gsc, ref, sub, rows)
    out = res.out.reshape(wl.B * T, wl.H, -1)[glob_rows]
    lse = res.lse.reshape(wl.B * T, wl.H)[glob_rows]
    check_mla(out, lse, gidx, sub, rows)
    if short and not staged:
        fused = api.decode_step(inp)
        torch.cuda.synchronize()
        assert int(fused.status.item()) == 0, _lib_status(fused.status)
        check_mla(fused.out.reshape(wl.B, wl.H, -1)[glob_rows], fused.lse.reshape(wl.B, wl.H)[glob_rows], gidx, sub,
                  rows)
    return res, inp


def _lib_status(st):
    from sparse_attention_04_b200 import _lib
    return _lib.status_string(int(st.item()))


# ------------------------------------------------------------------ small cases (full check)

def test_tiny_workload(cuda_device):
    run_and_check(dsa_inputs.WORKLOADS["tiny"], cuda_device)


@pytest.mark.parametrize("eps,k,H", [([1, 200, 777], 64, 16), ([40], 64, 16), ([300], 50, 16),
                                     ([600, 129, 128], 256, 128), ([2500, 3000], 2048, 128)])
def test_decode_ragged_batches(cuda_device, eps, k, H):
    wl = dsa_inputs.custom("ragged", B=len(eps), end_pos=None, topk=k, H=H, out_dtype="f32", seed=5,
                           end_pos_range=(1, 1))
    run_and_check(wl, cuda_device, end_pos=eps)


@pytest.mark.parametrize("T,eps,k", [(8, [8], 4), (300, [300], 64), (5, [50, 140], 16), (130, [400], 2048)])
def test_prefill_causal(cuda_device, T, eps, k):
    wl = dsa_inputs.custom("prefill", B=len(eps), T=T, end_pos=None, topk=k, H=128, out_dtype="bf16",
                           scale=192 ** -0.5, seed=7, end_pos_range=(1, 1))
    run_and_check(wl, cuda_device, end_pos=eps)


def test_decode_many_chunks_per_cta(cuda_device):
    """40 sequences, k=512: several 32-key chunks per attention CTA, each
    attention CTA's two gather stages cycling through its list."""
    wl = dsa_inputs.custom("many_chunks", B=40, end_pos=None, end_pos_range=(600, 3000), topk=512, H=128,
                           out_dtype="bf16", scale=192 ** -0.5, seed=21)
    run_and_check(wl, cuda_device, seqs=[0, 7, 23, 39])


def test_prefill_many_chunks_per_cta(cuda_device):
    """Causal prefill of 100 rows with k=512 (several chunks per CTA), with
    rows before, at and after the point where the causal prefix reaches k."""
    wl = dsa_inputs.custom("prefill_pg", B=1, T=100, end_pos=None, topk=512, H=128, out_dtype="bf16",
                           scale=192 ** -0.5, seed=22)
    run_and_check(wl, cuda_device, end_pos=[560], rows=[0, 1, 49, 50, 51, 52, 98, 99])


def test_short_context_skips_selection(cuda_device):
    """Every end_pos <= k: the decode step skips the indexer and the selection
    (all positions are kept whatever the scores) and attends to each whole
    prefix; the result must equal the oracle on the full index list."""
    api = _api()
    wl = dsa_inputs.custom("short", B=3, end_pos=None, topk=2048, H=128, out_dtype="bf16", scale=192 ** -0.5,
                           seed=31)
    inp = dsa_inputs.make_inputs(wl, cuda_device, end_pos=[100, 1500, 2048])
    res = api.decode_step(inp)
    torch.cuda.synchronize()
    assert int(res.status.item()) == 0, _lib_status(res.status)
    sub = subset(inp, [0, 1, 2])
    full = torch.full((3, 2048), -1, dtype=torch.int32)
    for b, E in enumerate(sub.end_pos):
        full[b, :E] = torch.arange(E, dtype=torch.int32)
    check_mla(res.out.reshape(3, wl.H, -1), res.lse.reshape(3, wl.H), full, sub, [0, 1, 2])


def test_short_context_many_rows(cuda_device):
    """The short-context path with enough rows that every attention CTA works
    through many chunks (the 64-key attention kernel), ragged prefixes."""
    api = _api()
    wl = dsa_inputs.custom("short_wide", B=24, end_pos=None, topk=2048, H=128, out_dtype="bf16", scale=192 ** -0.5,
                           seed=32)
    g = torch.Generator().manual_seed(33)
    eps = [int(x) for x in torch.randint(64, 2049, (24,), generator=g)]
    eps[0], eps[1], eps[2] = 1, 2048, 65
    inp = dsa_inputs.make_inputs(wl, cuda_device, end_pos=eps)
    res = api.decode_step(inp)
    torch.cuda.synchronize()
    assert int(res.status.item()) == 0, _lib_status(res.status)
    rows = [0, 1, 2, 13, 23]
    sub = subset(inp, rows)
    full = torch.full((len(rows), 2048), -1, dtype=torch.int32)
    for i, E in enumerate(sub.end_pos):
        full[i, :E] = torch.arange(E, dtype=torch.int32)
    out = res.out.reshape(24, wl.H, -1)[rows]
    lse = res.lse.reshape(24, wl.H)[rows]
    check_mla(out, lse, full, sub, list(range(len(rows))))


@pytest.mark.parametrize("B", [2, 20])  # 20 rows x 32 chunks of 64 take the 64-key kernel
def test_attention_on_arbitrary_index_lists(cuda_device, B):
    """dsa_sparse_mla on index lists it did not get from the selection:
    unsorted, with repeats, -1 holes, a whole 64-slot block of -1 ahead of
    valid slots, and one row with nothing selected (out 0, lse -inf)."""
    from sparse_attention_04_b200 import _lib
    k, H = 2048, 128
    wl = dsa_inputs.custom("arb_idx", B=B, end_pos=None, end_pos_range=(2500, 6000), topk=k, H=H,
                           out_dtype="bf16", scale=192 ** -0.5, seed=61)
    inp = dsa_inputs.make_inputs(wl, cuda_device)
    g = torch.Generator().manual_seed(62)
    idx = torch.stack([torch.randint(0, E, (k,), generator=g, dtype=torch.int32) for E in inp.end_pos])
    idx[torch.rand(B, k, generator=g) < 0.1] = -1
    idx[:, 128:192] = -1
    idx[:, :64] = -1  # the first chunk of every row holds nothing
    idx[B - 1] = -1
    idx = idx.to(cuda_device)
    out = torch.empty(B, 1, H, 512, dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty(B, 1, H, dtype=torch.float32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ws = torch.empty(max(16, _lib.sparse_mla_workspace_size(B, 1, H, k)), dtype=torch.uint8, device=cuda_device)
    _lib.sparse_mla(inp.q, inp.kv, inp.offsets, idx, B, 1, H, k, wl.scale, inp.rows, out, lse=lse, workspace=ws,
                    status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, _lib_status(st)
    seqs = [0, B - 1] if B == 2 else [0, 11, B - 1]
    sub = subset(inp, seqs)
    check_mla(out.reshape(B, H, -1)[seqs], lse.reshape(B, H)[seqs], idx[seqs], sub, list(range(len(seqs))))
    assert torch.all(out[B - 1] == 0) and torch.all(torch.isinf(lse[B - 1]) & (lse[B - 1] < 0))


def test_decode_mixed_lengths_long_pitch(cuda_device):
    """One decode step over rows of 5 to 70000 positions (score pitch above
    8192, so the selection runs as 4-CTA clusters): rows that keep every
    position sit beside rows that select, and the attention's splits of the
    short rows hold few or no chunks."""
    wl = dsa_inputs.custom("mixed", B=5, end_pos=None, topk=2048, H=16, out_dtype="bf16", scale=192 ** -0.5,
                           seed=63, end_pos_range=(1, 1))
    run_and_check(wl, cuda_device, end_pos=[5, 2000, 9000, 40000, 70000])


def test_fp8_small(cuda_device):
    wl = dsa_inputs.custom("fp8s", B=2, end_pos=None, topk=128, H=128, idx_dtype="e4m3", out_dtype="bf16",
                           scale=192 ** -0.5, seed=9, end_pos_range=(1, 1))
    run_and_check(wl, cuda_device, end_pos=[500, 1000])


def test_ties_follow_lower_position_first(cuda_device):
    """Duplicate key rows give exactly equal scores; the selection must keep the
    lowest positions among the tied ones, exactly as the oracle does."""
    def dup(inp):
        inp.k_idx[1::3] = inp.k_idx[0]
        inp.k_idx[2::7] = inp.k_idx[5]
    wl = dsa_inputs.custom("ties", B=1, end_pos=None, topk=100, H=16, out_dtype="f32", seed=11,
                           end_pos_range=(1, 1))
    run_and_check(wl, cuda_device, end_pos=[1000], mutate=dup)


def test_deterministic(cuda_device):
    api = _api()
    inp = dsa_inputs.make_inputs(dsa_inputs.custom("det", B=2, end_pos=5000, topk=512, H=128,
                                                   out_dtype="bf16", seed=13), cuda_device)
    a = api.decode_step(inp)
    o1, i1 = a.out.clone(), a.indices.clone()
    b = api.decode_step(inp)
    assert torch.equal(o1, b.out) and torch.equal(i1, b.indices)


# ------------------------------------------------------------------ full-size workloads (sampled)

def test_decode32k_full(cuda_device):
    run_and_check(dsa_inputs.WORKLOADS["decode32k"], cuda_device)


def test_batched_sampled(cuda_device):
    wl = dsa_inputs.WORKLOADS["batched"]
    run_and_check(wl, cuda_device, seqs=[0, 13, 31])


def test_prefill4k_sampled(cuda_device):
    wl = dsa_inputs.WORKLOADS["prefill4k"]
    rows = [0, 1, 127, 128, 129, 2046, 2047, 2048, 3000, 4095]
    run_and_check(wl, cuda_device, rows=rows)


def test_fp8_sampled(cuda_device):
    run_and_check(dsa_inputs.WORKLOADS["fp8"], cuda_device, seqs=[0, 3])
