"""Indexer pre-stage (rotary embedding of the rope half, then the Hadamard
rotation) through the C ABI, against the oracle.

Both sides round to bf16 at the same two points.  The kernel adds fp32
rounding before each of them, so an output can land one bf16 step away from
the oracle's when the exact value sits next to a rounding boundary: the test
allows one step there and checks that such cases are rare, and bounds every
output against the unrounded oracle by the error the two rounding points
allow."""
import math

import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _tables(n_pos, dev, base=10000.0):
    theta = base ** (-torch.arange(32, dtype=torch.float64) / 32)
    ang = torch.arange(n_pos, dtype=torch.float64)[:, None] * theta[None]
    return torch.cos(ang).float().to(dev), torch.sin(ang).float().to(dev)


def _ulp_bf16(x):
    """Spacing of bf16 values at |x| (fp64)."""
    e = torch.floor(torch.log2(x.abs().clamp_min(1e-30)))
    return torch.pow(2.0, e - 7)


def _check(x, pos, c, s, y):
    ref = oracle.rope_hadamard(x.cpu(), pos.cpu(), c.cpu(), s.cpu(), round_bf16=True)
    exact = oracle.rope_hadamard(x.cpu(), pos.cpu(), c.cpu(), s.cpu(), round_bf16=False)
    got = y.cpu().double()
    diff = (got - ref).abs()
    assert bool((diff <= _ulp_bf16(ref) * 1.0001 + 1e-30).all()), float(diff.max())
    assert float((diff > 0).double().mean()) < 0.02
    rope_l1 = x.cpu()[..., :64].double().abs().sum(-1, keepdim=True) * 1.42
    bound = 2.0 ** -7 * exact.abs() + 2.0 ** -8 * rope_l1 / math.sqrt(128) + 1e-12
    assert bool(((got - exact).abs() <= bound).all())


@pytest.mark.parametrize("n_rows,V", [(37, 64), (300, 1), (1, 1)])
def test_prestage_matches_oracle(cuda_device, n_rows, V):
    from sparse_attention_04_b200 import _lib
    g = torch.Generator(device=cuda_device).manual_seed(60 + V)
    L = 4096
    c, s = _tables(L, cuda_device)
    x = torch.randn(n_rows, V, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    pos = torch.randint(0, L, (n_rows,), generator=g, device=cuda_device, dtype=torch.int32)
    pos[0] = 0
    if n_rows > 1:
        pos[-1] = L - 1
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    y = _lib.indexer_prestage(x, pos, c, s, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check(x, pos, c, s, y)


def test_prestage_in_place_and_special_vectors(cuda_device):
    from sparse_attention_04_b200 import _lib
    g = torch.Generator(device=cuda_device).manual_seed(64)
    c, s = _tables(64, cuda_device)
    x = torch.randn(4, 8, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    x[0, 0] = 0                      # zero vector -> zero
    x[1, 1] = 0
    x[1, 1, 64] = 1.0                # a non-rope basis vector -> +-128^-1/2 everywhere
    pos = torch.tensor([0, 5, 17, 63], dtype=torch.int32, device=cuda_device)
    x0 = x.clone()
    _lib.indexer_prestage(x, pos, c, s, y=x)  # in place
    torch.cuda.synchronize()
    assert torch.equal(x[0, 0].float(), torch.zeros(128, device=cuda_device))
    assert torch.allclose(x[1, 1].float().abs(), torch.full((128,), 128 ** -0.5, device=cuda_device), rtol=2 ** -8)
    _check(x0, pos, c, s, x)


def test_prestage_rejects_bad_positions_and_arguments(cuda_device):
    from sparse_attention_04_b200 import _lib
    c, s = _tables(16, cuda_device)
    x = torch.randn(3, 2, 128, device=cuda_device).to(torch.bfloat16)
    pos = torch.tensor([1, 16, 2], dtype=torch.int32, device=cuda_device)  # row 1 is outside the table
    y = torch.full_like(x, 7.0)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _lib.indexer_prestage(x, pos, c, s, y=y, status=st)
    torch.cuda.synchronize()
    assert _lib.status_string(int(st.item())).startswith("DSA_ERR_BAD_INDEX")
    assert bool((y[1] == 7.0).all())                 # the bad row is untouched
    assert not bool((y[0] == 7.0).all()) and not bool((y[2] == 7.0).all())
    with pytest.raises(_lib.DSAError):
        _lib.indexer_prestage(x[:, :, :64].contiguous(), pos, c, s)
