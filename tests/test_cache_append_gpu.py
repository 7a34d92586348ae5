"""Cache write of the newest tokens and act_quant of the queries, through the
C ABI, against the oracle: integer work, so codes, scales and copied rows are
compared bit for bit (the quantiser's rule -- amax/448 scale in fp32, nearest
e4m3 code with ties to even, saturating -- is pinned in test_oracle.py)."""
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _caches(dev, rows, fp8, g):
    kv = torch.randn(rows, 576, generator=g, device=dev).to(torch.bfloat16)
    if fp8:
        k = torch.randint(0, 255, (rows, 128), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
        ks = torch.rand(rows, generator=g, device=dev)
    else:
        k = torch.randn(rows, 128, generator=g, device=dev).to(torch.bfloat16)
        ks = None
    return k, ks, kv


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("T", [1, 4])
def test_append_writes_exactly_the_last_rows(cuda_device, fp8, T):
    from sparse_attention_04_b200 import _lib
    g = torch.Generator(device=cuda_device).manual_seed(40 + T + 2 * fp8)
    eps = [7, 300, 64, 1]
    eps = [max(e, T) for e in eps]
    B = len(eps)
    off = torch.tensor([0] + list(torch.tensor(eps).cumsum(0)), dtype=torch.int32, device=cuda_device)
    rows = int(off[-1]) + 5  # slack rows after the last sequence stay untouched
    k, ks, kv = _caches(cuda_device, rows, fp8, g)
    k0, kv0 = k.clone(), kv.clone()
    ks0 = None if ks is None else ks.clone()
    # magnitudes over many binades, a zero vector, and exact ties after scaling
    k_new = (torch.randn(B, T, 128, generator=g, device=cuda_device) *
             torch.logspace(-3, 3, B * T, device=cuda_device).view(B, T, 1)).to(torch.bfloat16)
    k_new[0, 0] = 0
    kv_new = torch.randn(B, T, 576, generator=g, device=cuda_device).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _lib.cache_append(k_new, kv_new, off, B, T, k, ks, kv, rows, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    target = torch.cat([torch.arange(int(off[b + 1]) - T, int(off[b + 1])) for b in range(B)]).to(cuda_device)
    keep = torch.ones(rows, dtype=torch.bool, device=cuda_device)
    keep[target] = False
    assert torch.equal(kv[keep], kv0[keep]) and torch.equal(k[keep], k0[keep])
    assert torch.equal(kv[target].view(torch.int16), kv_new.reshape(-1, 576).view(torch.int16))
    if fp8:
        codes, scales = oracle.quantize_blocks(k_new.reshape(-1, 128).cpu())
        assert torch.equal(k[target].cpu(), codes)
        assert torch.equal(ks[target].cpu(), scales)
        assert torch.equal(ks[keep], ks0[keep])
    else:
        assert torch.equal(k[target].view(torch.int16), k_new.reshape(-1, 128).view(torch.int16))


def test_quantize_queries_codes_and_folded_weights(cuda_device):
    from sparse_attention_04_b200 import _lib
    g = torch.Generator(device=cuda_device).manual_seed(50)
    n_rows = 37
    q = (torch.randn(n_rows, 64, 128, generator=g, device=cuda_device) *
         torch.logspace(-2, 2, n_rows * 64, device=cuda_device).view(n_rows, 64, 1)).to(torch.bfloat16)
    q[3, 5] = 0
    w = torch.randn(n_rows, 64, generator=g, device=cuda_device) * (64 ** -0.5) * (128 ** -0.5)
    q8 = torch.empty(n_rows, 64, 128, dtype=torch.uint8, device=cuda_device)
    w_out = torch.empty_like(w)
    _lib.quantize_queries(q, w, n_rows, q8, w_out)
    torch.cuda.synchronize()
    codes, scales = oracle.quantize_blocks(q.cpu())
    assert torch.equal(q8.cpu(), codes)
    assert torch.equal(w_out.cpu(), w.cpu() * scales)  # one fp32 multiply, as Indexer.forward folds it


def test_append_reports_offsets_beyond_the_cache(cuda_device):
    from sparse_attention_04_b200 import _lib
    g = torch.Generator(device=cuda_device).manual_seed(51)
    rows = 64
    k, ks, kv = _caches(cuda_device, rows, False, g)
    k0, kv0 = k.clone(), kv.clone()
    off = torch.tensor([0, 10, 80], dtype=torch.int32, device=cuda_device)  # sequence 1 ends past kv_rows
    k_new = torch.randn(2, 1, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    kv_new = torch.randn(2, 1, 576, generator=g, device=cuda_device).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _lib.cache_append(k_new, kv_new, off, 2, 1, k, None, kv, rows, status=st)
    torch.cuda.synchronize()
    assert _lib.status_string(int(st.item())).startswith("DSA_ERR_BAD_OFFSETS")
    assert torch.equal(kv[9].view(torch.int16), kv_new[0, 0].view(torch.int16))  # the valid sequence is written
    mask = torch.ones(rows, dtype=torch.bool, device=cuda_device)
    mask[9] = False
    assert torch.equal(kv[mask], kv0[mask]) and torch.equal(k[mask], k0[mask])
