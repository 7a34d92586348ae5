"""dsa_topk on constructed score rows, bit-exact against the oracle's selection
(larger score first, then lower position; -0.0 == +0.0; ascending output, -1
padding).  Covers both the bitmap path and its fallback (threshold bin with
more candidates than the buffer, rows longer than the bitmap)."""
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _run(rows, k, T=1):
    """rows: list of 1-D float32 CPU tensors, one per sequence (T=1 decode rows)."""
    from sparse_attention_04_b200 import _lib
    dev = torch.device("cuda:0")
    eps = [r.numel() for r in rows]
    ld = (max(eps) + 3) // 4 * 4
    sc = torch.full((len(rows), ld), float("nan"), dtype=torch.float32)
    for i, r in enumerate(rows):
        sc[i, :r.numel()] = r
    off = torch.tensor([0] + list(torch.tensor(eps).cumsum(0).tolist()), dtype=torch.int32)
    out = torch.empty((len(rows), k), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    _lib.topk(sc.to(dev), ld, off.to(dev), len(rows), T, k, out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    want = oracle.topk(sc.double(), off, len(rows), T, k)
    return out.cpu(), want


def _gen(n, seed):
    return torch.randn(n, generator=torch.Generator().manual_seed(seed))


@pytest.mark.parametrize("n,k", [(32768, 2048), (32768 + 7, 2048), (131072, 2048), (131072 + 5, 2048),
                                 (5000, 4), (2049, 2048), (70000, 1)])
def test_random_rows(cuda_device, n, k):
    got, want = _run([_gen(n, n)], k)
    assert torch.equal(got, want)


def test_massive_ties_take_the_fallback(cuda_device):
    got, want = _run([torch.full((40000,), 0.5), torch.zeros(9000)], 2048)
    assert torch.equal(got, want)
    assert got[0].tolist() == list(range(2048))


def test_signed_zeros_and_few_distinct_values(cuda_device):
    g = torch.Generator().manual_seed(3)
    alphabet = torch.tensor([-0.0, 0.0, 1.0, -1.0, 2.5, 1e-30, -1e-30, float("-inf")])
    rows = [alphabet[torch.randint(0, 8, (30000,), generator=g)],
            torch.randn(30000, generator=g).round(decimals=1),     # ~60 distinct values, heavy ties
            torch.randn(12345, generator=g) * 1e-20]
    got, want = _run(rows, 2048)
    assert torch.equal(got, want)


def test_batch_of_ragged_rows(cuda_device):
    rows = [_gen(n, 100 + n) for n in (1, 31, 32, 33, 2047, 2048, 2049, 4096, 50000)]
    got, want = _run(rows, 2048)
    assert torch.equal(got, want)


@pytest.mark.parametrize("k", [1, 4, 2047, 2048])
def test_short_rows(cuda_device, k):
    """Rows of at most 8192 positions (one 256-thread CTA per row, keys held
    in registers): random rows, heavy ties, signed zeros and -inf, and ragged
    lengths around word and block boundaries."""
    g = torch.Generator().manual_seed(70 + k)
    alphabet = torch.tensor([-0.0, 0.0, 1.0, -1.0, 2.5, 1e-30, -1e-30, float("-inf")])
    rows = [_gen(n, 200 + n) for n in (2049, 2080, 4096, 5000, 8191, 8192)]
    rows += [alphabet[torch.randint(0, 8, (7000,), generator=g)], torch.full((6000,), 0.25),
             torch.randn(8000, generator=g).round(decimals=1), torch.randn(3000, generator=g) * 1e-20, _gen(5, 9)]
    got, want = _run(rows, k)
    assert torch.equal(got, want)


def test_causal_prefill_rows(cuda_device):
    """T = 600 query rows of one 6000-position sequence: row t keeps the top
    k of its causal prefix of 5401 + t positions."""
    from sparse_attention_04_b200 import _lib
    dev = torch.device("cuda:0")
    T, E, k = 600, 6000, 2048
    ld = E
    sc = torch.randn(T, ld, generator=torch.Generator().manual_seed(71))
    sc[::7] = sc[::7].round(decimals=1)  # some rows full of ties
    off = torch.tensor([0, E], dtype=torch.int32)
    out = torch.empty((T, k), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    _lib.topk(sc.to(dev), ld, off.to(dev), 1, T, k, out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out.cpu(), oracle.topk(sc.double(), off, 1, T, k))


@pytest.mark.parametrize("k", [1, 37, 2048])
def test_short_rows_16_keys_per_thread(cuda_device, k):
    """Rows of at most 4096 positions take 16 keys per thread: random rows,
    heavy ties, signed zeros and -inf, ragged lengths around the 16-key
    groups."""
    g = torch.Generator().manual_seed(90 + k)
    alphabet = torch.tensor([-0.0, 0.0, 1.0, -1.0, 2.5, 1e-30, -1e-30, float("-inf")])
    rows = [_gen(n, 300 + n) for n in (2049, 2065, 3000, 4095, 4096)]
    rows += [alphabet[torch.randint(0, 8, (4000,), generator=g)], torch.full((3500,), -0.5),
             torch.randn(4096, generator=g).round(decimals=1), _gen(17, 3)]
    got, want = _run(rows, k)
    assert torch.equal(got, want)
