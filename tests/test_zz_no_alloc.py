"""dsa_sparse_mla_noalloc: the sparse-MLA stage for callers that cannot
allocate device memory where they issue it (a plugin inside a runtime that owns
all device memory, a serving loop whose memory is fixed at start-up).  It keeps
its split partials in the library's own fixed scratch array instead of a
caller workspace, so these checks compare it with dsa_sparse_mla given a
workspace, on the same inputs, within the attention tolerance the other tests
use (|d| <= 1e-2 + 1e-2 |ref|), on two calls in a row (the scratch keeps the
previous call's contents, which must not leak into the next result).

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import pytest
import torch

from sparse_attention_04_b200 import inputs as dsa_inputs

pytestmark = pytest.mark.gpu


def _case(device, B, E, seed):
    wl = dsa_inputs.custom("noalloc", B=B, end_pos=E, topk=2048, H=128, out_dtype="bf16",
                           scale=192 ** -0.5, seed=seed)
    inp = dsa_inputs.make_inputs(wl, device)
    g = torch.Generator(device=device).manual_seed(seed)
    idx = torch.stack([torch.sort(torch.randperm(E, generator=g, device=device)[:2048]).values
                       for _ in range(B)]).to(torch.int32).contiguous()
    return wl, inp, idx


def _close(got, ref):
    g, r = got.double(), ref.double()
    return bool(torch.all((g - r).abs() <= 1e-2 + 1e-2 * r.abs()))


@pytest.mark.parametrize("B,E", [(1, 32768), (4, 9000)])
def test_noalloc_matches_workspace_entry_point_twice(cuda_device, B, E):
    from sparse_attention_04_b200 import _lib
    wl, inp, idx = _case(cuda_device, B, E, seed=B)
    assert _lib.sparse_mla_workspace_size(B, 1, 128, 2048) > 0  # this case does use scratch
    ref = torch.empty((B, 1, 128, 512), dtype=torch.bfloat16, device=cuda_device)
    ref_lse = torch.empty((B, 1, 128), dtype=torch.float32, device=cuda_device)
    ws = torch.empty(_lib.sparse_mla_workspace_size(B, 1, 128, 2048), dtype=torch.uint8, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _lib.sparse_mla(inp.q, inp.kv, inp.offsets, idx, B, 1, 128, 2048, wl.scale, inp.rows, ref, lse=ref_lse,
                    workspace=ws, status=st)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        _lib.sparse_mla_noalloc(inp.q, inp.kv, inp.offsets, idx, B, 1, 128, 2048, wl.scale, inp.rows, out,
                                lse=lse, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert _close(out, ref), f"call {call}: output differs"
        assert _close(lse, ref_lse), f"call {call}: lse differs"


def test_noalloc_rejects_work_beyond_its_scratch(cuda_device):
    from sparse_attention_04_b200 import _lib
    # a row count whose split partials exceed the built-in 32 MiB
    limit = 32 << 20
    rows = next(r for r in range(1, 4096) if _lib.sparse_mla_workspace_size(r, 1, 128, 2048) > limit)
    dummy = torch.zeros(16, dtype=torch.uint8, device=cuda_device)
    rc = _lib.lib.dsa_sparse_mla_noalloc(_lib._p(dummy), _lib._p(dummy), _lib._p(dummy), _lib._p(dummy), rows, 1,
                                         128, 2048, 0.1, 1 << 20, _lib._p(dummy), 0, None, None, None)
    assert rc == 3  # DSA_ERR_WORKSPACE, returned before anything is launched
