"""More parity cases of the CUDA path against the fp64 oracle, and the
device-side timeout path.

  - the e4m3 indexer with T > 1 (causal prefill rows of ragged sequences);
  - the attention at head counts other than 16 and 128, both output types;
  - the combine with several heads per CTA (a partly filled last group);
  - the pair kernel with fp32 output;
  - split rows on a workspace that starts zero, all ones or random, reused;
  - a short-context decode step whose query was written by the kernel copy
    just before it on the same stream;
  - a pipeline wait that runs out (test hook), then a normal call.

Tolerances are those of test_parity_gpu.py: scores 1e-3 * (1 + |ref|),
top-k bit-exact on the GPU's scores, attention 1e-2 + 1e-2 * |ref|.
"""
import pytest
import torch

import oracle
from sparse_attention_04_b200 import inputs as dsa_inputs

from test_parity_gpu import _lib_status, check_mla, run_and_check, subset

pytestmark = pytest.mark.gpu


def _lib():
    from sparse_attention_04_b200 import _lib as L
    return L


def _api():
    from sparse_attention_04_b200 import api
    return api


# ------------------------------------------------------------------ e4m3 indexer, T > 1

@pytest.mark.parametrize("T,eps,k", [(200, [300, 200], 64), (130, [129 + 130, 400], 128)])
def test_fp8_indexer_causal_prefill(cuda_device, T, eps, k):
    """e4m3 keys and queries (block scales) with T query rows per sequence:
    the prefill instance of the e4m3 indexer, causal mask, two ragged
    sequences; rows around a 128-key tile edge and each sequence's last row."""
    wl = dsa_inputs.custom("fp8_prefill", B=len(eps), T=T, end_pos=None, topk=k, H=16, idx_dtype="e4m3",
                           out_dtype="f32", scale=192 ** -0.5, seed=41, end_pos_range=(1, 1))
    local = [0, 1, 126, 127, 128, 129, T - 1]
    rows = sorted({b * T + t for b in range(len(eps)) for t in local if t < T})
    run_and_check(wl, cuda_device, end_pos=eps, rows=rows)


# ------------------------------------------------------------------ head counts

@pytest.mark.parametrize("H", [1, 5, 64, 100])
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_attention_head_counts(cuda_device, H, out_dtype):
    """dsa_sparse_mla at H outside {16, 128}: the query tile and the output
    boxes cover H rows per query row (the next row's heads, or zero fill past
    the end, on the query side).  Three rows, k = 2048 (splits and combine),
    plus a row with few selected positions."""
    L = _lib()
    B, k = 3, 2048
    wl = dsa_inputs.custom("heads", B=B, end_pos=None, end_pos_range=(2100, 5000), topk=k, H=H,
                           out_dtype=out_dtype, scale=192 ** -0.5, seed=50 + H)
    inp = dsa_inputs.make_inputs(wl, cuda_device)
    g = torch.Generator().manual_seed(51)
    idx = torch.stack([torch.randperm(E, generator=g)[:k].sort().values.to(torch.int32) for E in inp.end_pos])
    idx[1, 40:] = -1
    idx = idx.to(cuda_device)
    dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    out = torch.full((B, 1, H, 512), float("nan"), dtype=dt, device=cuda_device)
    lse = torch.empty(B, 1, H, dtype=torch.float32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ws = torch.empty(max(16, L.sparse_mla_workspace_size(B, 1, H, k)), dtype=torch.uint8, device=cuda_device)
    L.sparse_mla(inp.q, inp.kv, inp.offsets, idx, B, 1, H, k, wl.scale, inp.rows, out, lse=lse, workspace=ws,
                 status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, _lib_status(st)
    sub = subset(inp, list(range(B)))
    check_mla(out.reshape(B, H, -1), lse.reshape(B, H), idx, sub, list(range(B)))


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_combine_several_heads_per_cta(cuda_device, out_dtype):
    """32 rows at H = 100, k = 2048: two splits per row and a combine with
    eight heads per CTA, whose last group of each row holds four heads past
    H (they must write nothing).  Rows checked against the oracle; every
    output row must be finite."""
    L = _lib()
    B, H, k = 32, 100, 2048
    wl = dsa_inputs.custom("comb_g", B=B, end_pos=None, end_pos_range=(2100, 6000), topk=k, H=H,
                           out_dtype=out_dtype, scale=192 ** -0.5, seed=91)
    inp = dsa_inputs.make_inputs(wl, cuda_device)
    g = torch.Generator().manual_seed(92)
    idx = torch.stack([torch.randperm(E, generator=g)[:k].sort().values.to(torch.int32) for E in inp.end_pos])
    idx = idx.to(cuda_device)
    dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    out = torch.full((B + 1, 1, H, 512), float("nan"), dtype=dt, device=cuda_device)  # + a guard row
    lse = torch.full((B + 1, 1, H), float("nan"), dtype=torch.float32, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ws = torch.empty(max(16, L.sparse_mla_workspace_size(B, 1, H, k)), dtype=torch.uint8, device=cuda_device)
    L.sparse_mla(inp.q, inp.kv, inp.offsets, idx, B, 1, H, k, wl.scale, inp.rows, out[:B], lse=lse[:B],
                 workspace=ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, _lib_status(st)
    assert torch.isfinite(out[:B].float()).all() and torch.isfinite(lse[:B]).all()
    assert torch.isnan(out[B].float()).all() and torch.isnan(lse[B]).all()  # nothing written past the rows
    rows = [0, 13, 31]
    sub = subset(inp, rows)
    check_mla(out[rows].reshape(len(rows), H, -1), lse[rows].reshape(len(rows), H), idx[rows], sub,
              list(range(len(rows))))


@pytest.mark.parametrize("H", [1, 5, 64, 100])
def test_short_context_head_counts(cuda_device, H):
    """The decode step's dense short-context attention at the same head counts."""
    api = _api()
    wl = dsa_inputs.custom("short_heads", B=2, end_pos=None, topk=2048, H=H, out_dtype="f32",
                           scale=192 ** -0.5, seed=60 + H)
    inp = dsa_inputs.make_inputs(wl, cuda_device, end_pos=[700, 2048])
    res = api.decode_step(inp)
    torch.cuda.synchronize()
    assert int(res.status.item()) == 0, _lib_status(res.status)
    sub = subset(inp, [0, 1])
    full = torch.full((2, 2048), -1, dtype=torch.int32)
    for b, E in enumerate(sub.end_pos):
        full[b, :E] = torch.arange(E, dtype=torch.int32)
    check_mla(res.out.reshape(2, H, -1), res.lse.reshape(2, H), full, sub, [0, 1])


# ------------------------------------------------------------------ pair kernel, fp32 output

def test_pair_kernel_fp32_output(cuda_device):
    """160 causal prefill rows, k = 2048: enough 128-key chunks for the
    pair kernel (QK CTA + PV CTA), one unit per row, and fp32 output, which
    its epilogue writes in two 256-column passes through the value ring."""
    from test_parity_gpu import run_and_check as rc
    wl = dsa_inputs.custom("pair_f32", B=1, T=160, end_pos=None, topk=2048, H=128, out_dtype="f32",
                           scale=192 ** -0.5, seed=111, end_pos_range=(1, 1))
    rc(wl, cuda_device, end_pos=[400], rows=[0, 1, 2, 79, 158, 159])


# ------------------------------------------------------------------ split rows on a reused workspace

@pytest.mark.parametrize("fill", [0x00, 0xFF, None])
def test_split_rows_on_reused_workspace(cuda_device, fill):
    """Two 20K rows, k = 2048: the 64-key kernel splits each row 32 ways and
    the combine merges the partials.  The workspace starts all zero, all ones
    or random; three calls with different index lists then run on it back to
    back (the last with empty later splits), and each must match the oracle:
    nothing a call reads may come from what an earlier call left there."""
    L = _lib()
    B, H, k = 2, 128, 2048
    wl = dsa_inputs.custom("reuse_ws", B=B, end_pos=20000, topk=k, H=H, out_dtype="bf16",
                           scale=192 ** -0.5, seed=101)
    inp = dsa_inputs.make_inputs(wl, cuda_device)
    nbytes = L.sparse_mla_workspace_size(B, 1, H, k)
    assert nbytes > 0
    if fill is None:
        ws = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=torch.Generator().manual_seed(3))
        ws = ws.to(cuda_device)
    else:
        ws = torch.full((nbytes,), fill, dtype=torch.uint8, device=cuda_device)
    sub = subset(inp, [0, 1])
    g = torch.Generator().manual_seed(102)
    for call in range(3):
        idx = torch.stack([torch.randperm(E, generator=g)[:k].sort().values.to(torch.int32) for E in inp.end_pos])
        if call == 2:
            idx[1, 1000:] = -1  # later splits of row 1 hold nothing
        out = torch.full((B, 1, H, 512), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        lse = torch.empty(B, 1, H, dtype=torch.float32, device=cuda_device)
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        L.sparse_mla(inp.q, inp.kv, inp.offsets, idx.to(cuda_device), B, 1, H, k, wl.scale, inp.rows, out,
                     lse=lse, workspace=ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, _lib_status(st)
        check_mla(out.reshape(B, H, -1), lse.reshape(B, H), idx, sub, [0, 1])


# ------------------------------------------------------------------ ordering after a copy kernel

def test_short_context_step_after_query_copy_on_same_stream(cuda_device):
    """The query is written by dsa_copy_host_to_device immediately before a
    short-context dsa_decode_step on the same stream (no other library kernel
    in between): the attention must read the copied query, not what the
    buffer held before."""
    L, api = _lib(), _api()
    wl = dsa_inputs.custom("short_copy", B=2, end_pos=None, topk=2048, H=128, out_dtype="bf16",
                           scale=192 ** -0.5, seed=71)
    inp = dsa_inputs.make_inputs(wl, cuda_device, end_pos=[1500, 2048])
    host_q = torch.empty(inp.q.shape, dtype=torch.bfloat16, pin_memory=True)
    host_q.copy_(inp.q.cpu())
    step = api.DecodeStep(wl.B, max(inp.end_pos), wl.topk, wl.H, torch.bfloat16, cuda_device)
    q_dev = torch.empty_like(inp.q)
    sub = subset(inp, [0, 1])
    full = torch.full((2, 2048), -1, dtype=torch.int32)
    for b, E in enumerate(sub.end_pos):
        full[b, :E] = torch.arange(E, dtype=torch.int32)
    stream = torch.cuda.Stream(cuda_device)
    for rep in range(3):
        q_dev.fill_(-7.0 - rep)  # stale contents a premature read would see
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            L.copy_host_to_device(q_dev, host_q)
            step(inp.q_idx, inp.w, inp.k_idx, inp.k_scale, q_dev, inp.kv, inp.offsets, inp.rows, wl.scale)
        torch.cuda.synchronize()
        assert int(step.status.item()) == 0, _lib_status(step.status)
        check_mla(step.out.reshape(2, wl.H, -1), step.lse.reshape(2, wl.H), full, sub, [0, 1])


# ------------------------------------------------------------------ device timeout path

DSA_ERR_TIMEOUT = 5


@pytest.mark.parametrize("case", ["selection", "short_context"])
def test_pipeline_wait_runs_out_then_next_call_is_correct(cuda_device, case):
    """The test hook makes the next attention launch's query barrier expect
    one arrival that never comes, with a 5 ms wait limit.  The launch must end
    by itself and report DSA_ERR_TIMEOUT in the status word; the next call on
    the same stream (whose kernels allocate the same tensor memory again)
    must succeed and match the oracle."""
    L, api = _lib(), _api()
    if case == "selection":   # indexer -> selection -> 64-key attention kernel
        wl = dsa_inputs.WORKLOADS["tiny"]
        inp = dsa_inputs.make_inputs(wl, cuda_device)
    else:                     # dense short-context attention (32-key kernel for one row)
        wl = dsa_inputs.custom("short_stall", B=1, end_pos=None, topk=2048, H=128, out_dtype="bf16",
                               scale=192 ** -0.5, seed=81)
        inp = dsa_inputs.make_inputs(wl, cuda_device, end_pos=[1800])
    step = api.DecodeStep(wl.B, max(inp.end_pos), wl.topk, wl.H,
                          torch.float32 if wl.out_dtype == "f32" else torch.bfloat16, cuda_device)
    L.debug_stall_attention(1, 5_000_000)
    try:
        step(inp.q_idx, inp.w, inp.k_idx, inp.k_scale, inp.q, inp.kv, inp.offsets, inp.rows, wl.scale)
        torch.cuda.synchronize()
    finally:
        L.debug_stall_attention(0, 0)
    assert int(step.status.item()) == DSA_ERR_TIMEOUT, _lib_status(step.status)
    step.status.zero_()
    step(inp.q_idx, inp.w, inp.k_idx, inp.k_scale, inp.q, inp.kv, inp.offsets, inp.rows, wl.scale)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0, _lib_status(step.status)
    sub = subset(inp, [0])
    E = sub.end_pos[0]
    if case == "selection":
        ref = oracle.indexer_scores(sub.q_idx, sub.w, sub.k_idx, None, sub.offsets, 1, 1, E)
        sel = oracle.topk(step.scores[:, :E].double().cpu(), sub.offsets, 1, 1, wl.topk)
        assert torch.equal(sel, step.indices.cpu())
        assert torch.all((step.scores[:, :E].double().cpu() - ref).abs() <= 1e-3 * (1 + ref.abs()))
    else:
        sel = torch.full((1, wl.topk), -1, dtype=torch.int32)
        sel[0, :E] = torch.arange(E, dtype=torch.int32)
    check_mla(step.out.reshape(1, wl.H, -1), step.lse.reshape(1, wl.H), sel, sub, [0])
