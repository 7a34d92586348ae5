"""Kernel-driven copies between pinned host memory and the device
(dsa_copy_host_to_device / dsa_copy_device_to_host): bit-exact round trips
over ragged sizes, fresh host data on every replay of a captured graph (no
stale cached lines), and the host-side rejection of buffers the kernels may
not touch."""
import ctypes

import pytest
import torch

from sparse_attention_04_b200 import _lib

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _pinned_bytes(n, seed):
    g = torch.Generator().manual_seed(seed)
    t = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    t.copy_(torch.randint(0, 256, (n,), generator=g, dtype=torch.uint8))
    return t


@pytest.mark.parametrize("n", [16, 4096 + 48, 165632, 5_296_128 + 16])
def test_round_trip(n):
    src = _pinned_bytes(n, n)
    dev = torch.full((n,), 7, dtype=torch.uint8, device=DEV)
    _lib.copy_host_to_device(dev, src)
    torch.cuda.synchronize()
    assert torch.equal(dev.cpu(), src)
    back = torch.zeros(n, dtype=torch.uint8, pin_memory=True)
    _lib.copy_device_to_host(back, dev)
    torch.cuda.synchronize()
    assert torch.equal(back, src)


def test_graph_replays_see_new_host_data():
    n = 1 << 16
    src = _pinned_bytes(n, 1)
    out = torch.zeros(n, dtype=torch.uint8, pin_memory=True)
    dev = torch.empty(n, dtype=torch.uint8, device=DEV)
    stream = torch.cuda.Stream(DEV)
    with torch.cuda.stream(stream):
        _lib.copy_host_to_device(dev, src)
        _lib.copy_device_to_host(out, dev)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        _lib.copy_host_to_device(dev, src)
        dev.add_(1)
        _lib.copy_device_to_host(out, dev)
    for seed in (2, 3, 4):
        src.copy_(_pinned_bytes(n, seed))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, src + 1)


def test_rejects_unusable_host_buffers():
    dev = torch.empty(4096, dtype=torch.uint8, device=DEV)
    pageable = torch.zeros(4096, dtype=torch.uint8)
    with pytest.raises(_lib.DSAError) as e:
        _lib.copy_host_to_device(dev, pageable)
    assert e.value.code == 1
    with pytest.raises(_lib.DSAError) as e:
        _lib.copy_device_to_host(pageable, dev)
    assert e.value.code == 1
    pinned = torch.zeros(4096 + 16, dtype=torch.uint8, pin_memory=True)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    d = ctypes.c_void_p(dev.data_ptr())
    # ragged size, unaligned pointer: refused before any launch
    assert _lib.lib.dsa_copy_host_to_device(d, ctypes.c_void_p(pinned.data_ptr()), 4088, s) == 1
    assert _lib.lib.dsa_copy_host_to_device(d, ctypes.c_void_p(pinned.data_ptr() + 8), 4096, s) == 1
    # a range running far past the pinned allocation: its last byte is not mapped
    assert _lib.lib.dsa_copy_host_to_device(d, ctypes.c_void_p(pinned.data_ptr()), 1 << 40, s) == 1
    assert _lib.lib.dsa_copy_host_to_device(d, ctypes.c_void_p(pinned.data_ptr()), 0, s) == 0
    torch.cuda.synchronize()
