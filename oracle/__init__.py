"""fp64 oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  It wraps `dsa_oracle.c` (plain C loops in double precision,
built with gcc) through ctypes and shares no code with the CUDA library.

Functions take torch CPU tensors (the exact bytes the seeded input module
drew) and return float64 / int32 torch tensors.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

H_I, D_I, D_QK, D_V = 64, 128, 576, 512


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-Wall",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        _lib.oracle_indexer_scores.argtypes = [P, P, P, P, I, P, I, I, P, I64, P, I64, P]
        _lib.oracle_topk.argtypes = [P, I64, P, I, I, I, P, I64, P]
        _lib.oracle_sparse_mla.argtypes = [P, P, P, P, I, I, I, I, D, P, I64, P, P, P]
        _lib.oracle_dense_mla.argtypes = [P, P, P, I, I, I, D, P, I64, P, P, P]
        _lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        _lib.oracle_bf16_to_f64.restype = D
        _lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_to_f64.restype = D
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        _lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        _lib.oracle_quantize_blocks.argtypes = [P, I64, P, P]
        _lib.oracle_rope_hadamard.argtypes = [P, I64, I, P, P, P, I64, I, P]
        for f in ("oracle_indexer_scores", "oracle_topk", "oracle_sparse_mla", "oracle_dense_mla",
                  "oracle_num_threads", "oracle_quantize_blocks", "oracle_rope_hadamard"):
            getattr(_lib, f).restype = I
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous()
    return ctypes.c_void_p(t.data_ptr())


def _bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 -> uint16 bit view; uint8 (e4m3 codes) unchanged."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16)
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return t.view(torch.uint8)
    raise TypeError(t.dtype)


def _rows(rows: Optional[Sequence[int]]):
    if rows is None:
        return None, 0
    r = torch.tensor(list(rows), dtype=torch.int64)
    return r, r.numel()


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


class Counter:
    def __init__(self):
        self.c = ctypes.c_int64(0)

    @property
    def value(self):
        return int(self.c.value)


def indexer_scores(q_idx, w, k_idx, k_scale, offsets, B, T, ld, rows=None, macs: Counter = None):
    """fp64 indexer scores, [n_rows, ld]; entries past end_pos are NaN (not written)."""
    dtype = 0 if q_idx.dtype == torch.bfloat16 else 1
    r, n = _rows(rows)
    n_out = n if rows is not None else B * T
    out = torch.full((n_out, ld), float("nan"), dtype=torch.float64)
    qb, kb = _bits(q_idx), _bits(k_idx)
    wc = w.detach().cpu().float().contiguous()
    ks = None if k_scale is None else k_scale.detach().cpu().float().contiguous()
    off = offsets.detach().cpu().to(torch.int32).contiguous()
    rc = lib().oracle_indexer_scores(_ptr(qb), _ptr(wc), _ptr(kb), _ptr(ks), dtype, _ptr(off), B, T,
                                     _ptr(r), n, _ptr(out), ld,
                                     ctypes.byref(macs.c) if macs else None)
    _check(rc, "indexer_scores")
    return out


def topk(scores, offsets, B, T, k, rows=None):
    """Selection on a [n_rows, ld] score tensor (float32 or float64)."""
    sc = scores.detach().cpu().to(torch.float64).contiguous()
    r, n = _rows(rows)
    n_out = n if rows is not None else B * T
    assert sc.shape[0] == n_out
    out = torch.empty((n_out, k), dtype=torch.int32)
    off = offsets.detach().cpu().to(torch.int32).contiguous()
    rc = lib().oracle_topk(_ptr(sc), sc.shape[1], _ptr(off), B, T, k, _ptr(r), n, _ptr(out))
    _check(rc, "topk")
    return out


def sparse_mla(q, kv, offsets, indices, B, T, H, k, scale, rows=None, macs: Counter = None):
    """Returns (out [n_rows,H,512] f64, lse [n_rows,H] f64); indices [n_rows,k] int32."""
    r, n = _rows(rows)
    n_out = n if rows is not None else B * T
    idx = indices.detach().cpu().to(torch.int32).contiguous()
    assert idx.shape == (n_out, k)
    out = torch.empty((n_out, H, D_V), dtype=torch.float64)
    lse = torch.empty((n_out, H), dtype=torch.float64)
    off = offsets.detach().cpu().to(torch.int32).contiguous()
    rc = lib().oracle_sparse_mla(_ptr(_bits(q)), _ptr(_bits(kv)), _ptr(off), _ptr(idx), B, T, H, k,
                                 float(scale), _ptr(r), n, _ptr(out), _ptr(lse),
                                 ctypes.byref(macs.c) if macs else None)
    _check(rc, "sparse_mla")
    return out, lse


def dense_mla(q, kv, offsets, B, T, H, scale, rows=None, macs: Counter = None):
    r, n = _rows(rows)
    n_out = n if rows is not None else B * T
    out = torch.empty((n_out, H, D_V), dtype=torch.float64)
    lse = torch.empty((n_out, H), dtype=torch.float64)
    off = offsets.detach().cpu().to(torch.int32).contiguous()
    rc = lib().oracle_dense_mla(_ptr(_bits(q)), _ptr(_bits(kv)), _ptr(off), B, T, H, float(scale),
                                _ptr(r), n, _ptr(out), _ptr(lse),
                                ctypes.byref(macs.c) if macs else None)
    _check(rc, "dense_mla")
    return out, lse


def bf16_to_f64(bits: int) -> float:
    return lib().oracle_bf16_to_f64(bits)


def e4m3_to_f64(code: int) -> float:
    return lib().oracle_e4m3_to_f64(code)


def e4m3_encode(x: float) -> int:
    """Nearest e4m3 code to the fp32 value x (ties to even, saturating at +-448)."""
    return int(lib().oracle_e4m3_encode(float(x)))


def quantize_blocks(x) -> tuple:
    """act_quant of [..., 128] bf16 vectors: (uint8 codes [..., 128], fp32 scales [...])."""
    xb = _bits(x)
    assert x.shape[-1] == D_I
    n = xb.numel() // D_I
    codes = torch.empty(xb.shape, dtype=torch.uint8)
    scales = torch.empty(xb.shape[:-1], dtype=torch.float32)
    _check(lib().oracle_quantize_blocks(_ptr(xb), n, _ptr(codes), _ptr(scales)), "quantize_blocks")
    return codes, scales


def rope_hadamard(x, pos, rope_cos, rope_sin, round_bf16: bool = True):
    """Indexer pre-stage of [n_rows, V, 128] bf16 vectors (V vectors share a
    row's position pos[row]): rotary embedding of the first 64 entries (pairs
    i, i+32) with the [rope_len, 32] cos/sin tables, then the 128-point
    Hadamard rotation.  Returns float64 [n_rows, V, 128]; with round_bf16 the
    two bf16 rounding points of the model are applied (values exactly bf16)."""
    xb = _bits(x)
    assert x.dim() == 3 and x.shape[-1] == D_I
    n_rows, V = x.shape[0], x.shape[1]
    p = pos.detach().cpu().to(torch.int32).contiguous()
    c = rope_cos.detach().cpu().float().contiguous()
    s = rope_sin.detach().cpu().float().contiguous()
    assert p.numel() == n_rows and c.shape == s.shape and c.shape[1] == 32
    y = torch.empty((n_rows, V, D_I), dtype=torch.float64)
    _check(lib().oracle_rope_hadamard(_ptr(xb), n_rows, V, _ptr(p), _ptr(c), _ptr(s), c.shape[0],
                                      1 if round_bf16 else 0, _ptr(y)), "rope_hadamard")
    return y


def num_threads() -> int:
    return lib().oracle_num_threads()


def decode_step(inp, rows=None):
    """Whole path on the oracle's own scores: (scores f64, indices, out f64, lse f64)."""
    wl = inp.wl
    B, T = wl.B, wl.T
    ld = max(inp.end_pos)
    sc = indexer_scores(inp.q_idx, inp.w, inp.k_idx, inp.k_scale, inp.offsets, B, T, ld, rows=rows)
    idx = topk(sc, inp.offsets, B, T, wl.topk, rows=rows)
    out, lse = sparse_mla(inp.q, inp.kv, inp.offsets, idx, B, T, wl.H, wl.topk, wl.scale, rows=rows)
    return sc, idx, out, lse
