"""The host-fed decode step (api.HostDecodeStep): pinned host inputs in, the
cache write, the three stages, the output back in pinned host memory.

It must give exactly what the device-buffer path gives for the same inputs
(same kernels, same launch shapes: bit-identical caches, indices and output),
and its attention output is checked against the oracle on the updated caches
with the attention tolerance of the parity tests."""
import pytest
import torch

from sparse_attention_04_b200 import inputs as dsa_inputs
from sparse_attention_04_b200.inputs import Inputs
from test_parity_gpu import check_mla

pytestmark = pytest.mark.gpu


def _fill_host(hs, B, H, seed):
    g = torch.Generator().manual_seed(seed)
    hs.host_q_idx.copy_(torch.randn(B, 1, 64, 128, generator=g).to(torch.bfloat16))
    hs.host_w.copy_(torch.rand(B, 1, 64, generator=g) * 2 - 1)
    hs.host_q.copy_(torch.randn(B, 1, H, 576, generator=g).to(torch.bfloat16))
    hs.host_k_new.copy_(torch.randn(B, 1, 128, generator=g).to(torch.bfloat16))
    hs.host_kv_new.copy_(torch.randn(B, 1, 576, generator=g).to(torch.bfloat16))


# How q crosses PCIe depends on its size: with the small inputs (the first
# three cases), by a side-stream copy kernel after the indexer (the fourth,
# 295 KB), by the copy engine (the last, above HostDecodeStep.Q_KERNEL_COPY_MAX)
@pytest.mark.parametrize("idx_dtype,eps,k,H", [("bf16", [3000, 5000, 1500], 2048, 16), ("e4m3", [700, 1200], 256, 16),
                                               ("bf16", [100, 2048, 1], 2048, 16),
                                               ("bf16", [3000, 2500], 2048, 128),
                                               ("bf16", [900, 1300, 600, 1000, 700, 2000, 650, 1100], 512, 128)])
def test_host_step_matches_device_path_and_oracle(cuda_device, idx_dtype, eps, k, H):
    from sparse_attention_04_b200 import _lib, api
    B = len(eps)
    wl = dsa_inputs.custom("host_step", B=B, end_pos=None, topk=k, H=H, idx_dtype=idx_dtype, out_dtype="bf16",
                           seed=51, end_pos_range=(1, 1))
    inp = dsa_inputs.make_inputs(wl, cuda_device, end_pos=eps)
    k2, kv2 = inp.k_idx.clone(), inp.kv.clone()
    ks2 = None if inp.k_scale is None else inp.k_scale.clone()
    hs = api.HostDecodeStep(B, max(eps), k, H, idx_dtype, torch.bfloat16, cuda_device)
    q_bytes = B * H * 576 * 2  # the path the step takes for q, as the cases above intend
    path = "inputs" if q_bytes <= hs.Q_WITH_INPUTS_MAX else "kernel" if q_bytes <= hs.Q_KERNEL_COPY_MAX else "engine"
    assert path == ("inputs" if H == 16 else "kernel" if B == 2 else "engine") and hs.q_with_inputs == (path == "inputs")
    for seed in (1, 2):  # two calls: the second must see the refilled host inputs
        _fill_host(hs, B, H, 70 + seed)
        out = hs(inp.k_idx, inp.k_scale, inp.kv, inp.offsets, inp.rows, wl.scale)
        torch.cuda.synchronize()
        assert int(hs.step.status.item()) == 0, _lib.status_string(int(hs.step.status.item()))

        # the same step through device buffers
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        _lib.cache_append(hs.host_k_new.to(cuda_device), hs.host_kv_new.to(cuda_device), inp.offsets, B, 1, k2, ks2,
                          kv2, inp.rows, status=st)
        q_idx, w = hs.host_q_idx.to(cuda_device), hs.host_w.to(cuda_device)
        if idx_dtype == "e4m3":
            q8 = torch.empty(B, 1, 64, 128, dtype=torch.uint8, device=cuda_device)
            w8 = torch.empty(B, 1, 64, dtype=torch.float32, device=cuda_device)
            _lib.quantize_queries(q_idx, w, B, q8, w8)
            q_idx, w = q8, w8
        ds = api.DecodeStep(B, max(eps), k, H, torch.bfloat16, cuda_device)
        q = hs.host_q.to(cuda_device)
        ds(q_idx, w, k2, ks2, q, kv2, inp.offsets, inp.rows, wl.scale)
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(ds.status.item()) == 0
        assert torch.equal(inp.kv.view(torch.int16), kv2.view(torch.int16))
        assert torch.equal(inp.k_idx.view(torch.uint8), k2.view(torch.uint8))
        if ks2 is not None:
            assert torch.equal(inp.k_scale, ks2)
        short = max(eps) <= k
        if not short:
            assert torch.equal(hs.step.indices, ds.indices)
        assert torch.equal(out.view(torch.int16), ds.out.cpu().view(torch.int16))

        # the attention output against the oracle on the updated caches
        if short:
            idx = torch.full((B, k), -1, dtype=torch.int32)
            for b, E in enumerate(eps):
                idx[b, :E] = torch.arange(E, dtype=torch.int32)
        else:
            idx = hs.step.indices.cpu()
        sub = Inputs(wl, list(eps), inp.offsets.cpu(), None, None, None, None, hs.host_q.clone(), inp.kv.cpu())
        check_mla(out.reshape(B, H, -1), hs.step.lse.reshape(B, H), idx, sub, list(range(B)))


@pytest.mark.parametrize("H", [16, 128])
def test_host_step_in_a_cuda_graph(cuda_device, H):
    """Captured once, replayed with the host inputs refilled between
    replays: each replay's output matches an eager host-fed step on the same
    inputs and caches.  H = 16: q travels with the small inputs; H = 128
    (295 KB): by a side-stream copy kernel after the indexer."""
    from sparse_attention_04_b200 import api
    B, k = 2, 512
    eps = [9000, 3000]
    wl = dsa_inputs.custom("host_graph", B=B, end_pos=None, topk=k, H=H, out_dtype="bf16", seed=91,
                           end_pos_range=(1, 1))
    inp = dsa_inputs.make_inputs(wl, cuda_device, end_pos=eps)
    hs = api.HostDecodeStep(B, max(eps), k, H, "bf16", torch.bfloat16, cuda_device)
    ref_hs = api.HostDecodeStep(B, max(eps), k, H, "bf16", torch.bfloat16, cuda_device)
    kv2, k2 = inp.kv.clone(), inp.k_idx.clone()
    stream = torch.cuda.Stream(cuda_device)
    _fill_host(hs, B, H, 100)
    with torch.cuda.stream(stream):
        hs(inp.k_idx, inp.k_scale, inp.kv, inp.offsets, inp.rows, wl.scale)  # warm-up, outside the graph
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        hs(inp.k_idx, inp.k_scale, inp.kv, inp.offsets, inp.rows, wl.scale)
    for seed in (101, 102, 103):
        _fill_host(hs, B, H, seed)
        g.replay()
        torch.cuda.synchronize()
        assert int(hs.step.status.item()) == 0
        _fill_host(ref_hs, B, H, seed)
        ref = ref_hs(k2, None, kv2, inp.offsets, inp.rows, wl.scale)
        torch.cuda.synchronize()
        assert torch.equal(hs.host_out.view(torch.int16), ref.view(torch.int16))
