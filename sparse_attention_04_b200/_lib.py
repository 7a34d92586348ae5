"""ctypes binding of libdsa.so: argument marshalling only.

Every function below takes torch CUDA tensors, passes their device pointers
and the current CUDA stream to the C ABI of the same name (include/dsa.h) and
raises DSAError on a non-zero status.  No arithmetic of the method happens
here; there is no CPU fallback.  If libdsa.so is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_BF16, DSA_E4M3, DSA_F32 = 0, 1, 2
STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
          4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_BAD_INDEX", 7: "DSA_ERR_BAD_OFFSETS"}

EXPORTS = ("dsa_status_string", "dsa_version", "dsa_indexer_scores", "dsa_topk",
           "dsa_sparse_mla_workspace_size", "dsa_sparse_mla", "dsa_decode_step_workspace_size",
           "dsa_decode_step", "dsa_decode_step_workspace_layout", "dsa_sparse_mla_noalloc",
           "dsa_decode_step_launches", "dsa_cache_append", "dsa_quantize_queries", "dsa_indexer_prestage",
           "dsa_copy_host_to_device", "dsa_copy_device_to_host", "dsa_debug_stall_attention")


class DSAError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m sparse_attention_04_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "dsa_status_string": ([I], ctypes.c_char_p),
        "dsa_version": ([], I),
        "dsa_indexer_scores": ([P, P, P, P, I, P, I, I, I64, P, I64, P, P], I),
        "dsa_topk": ([P, I64, P, I, I, I, P, P, P], I),
        "dsa_sparse_mla_workspace_size": ([I, I, I, I], SZ),
        "dsa_sparse_mla": ([P, P, P, P, I, I, I, I, F, I64, P, I, P, P, SZ, P, P], I),
        "dsa_decode_step_workspace_size": ([I, I, I, I], SZ),
        "dsa_decode_step": ([P, P, P, P, I, P, P, P, I, I, I64, I, I, F, P, I, P, P, SZ, P, P], I),
        "dsa_decode_step_workspace_layout": ([I, I, I, I, P, P, P, P], I),
        "dsa_sparse_mla_noalloc": ([P, P, P, P, I, I, I, I, F, I64, P, I, P, P, P], I),
        "dsa_decode_step_launches": ([I, I, I, I], I),
        "dsa_cache_append": ([P, P, P, I, I, I, P, P, P, I64, P, P], I),
        "dsa_quantize_queries": ([P, P, I, P, P, P], I),
        "dsa_indexer_prestage": ([P, P, I, I, P, P, I, P, P, P], I),
        "dsa_copy_host_to_device": ([P, P, SZ, P], I),
        "dsa_copy_device_to_host": ([P, P, SZ, P], I),
        "dsa_debug_stall_attention": ([I, ctypes.c_uint64], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise DSAError(1, "tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise DSAError(1, "tensor is not contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise DSAError(rc, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_E4M3
    raise DSAError(1, f"unsupported indexer dtype {t.dtype}")


def status_string(code: int) -> str:
    return lib.dsa_status_string(code).decode()


def indexer_scores(q_idx, w, k_idx, k_scale, offsets, B, T, kv_rows, scores, ld, status=None, stream=None):
    """dsa_indexer_scores: writes fp32 scores[(b*T+t)*ld + s]."""
    _check(lib.dsa_indexer_scores(_p(q_idx), _p(w), _p(k_idx), _p(k_scale), _dtype_code(q_idx), _p(offsets),
                                  B, T, kv_rows, _p(scores), ld, _p(status), _stream(stream)),
           "dsa_indexer_scores")


def topk(scores, ld, offsets, B, T, k, indices, status=None, stream=None):
    """dsa_topk: int32 indices [B*T, k], ascending, -1 padded."""
    _check(lib.dsa_topk(_p(scores), ld, _p(offsets), B, T, k, _p(indices), _p(status), _stream(stream)),
           "dsa_topk")


def sparse_mla_workspace_size(B, T, H, k) -> int:
    return int(lib.dsa_sparse_mla_workspace_size(B, T, H, k))


def sparse_mla(q, kv, offsets, indices, B, T, H, k, scale, kv_rows, out, lse=None, workspace=None,
               status=None, stream=None):
    """dsa_sparse_mla: out [B,T,H,512] (bf16 or fp32 by out's dtype)."""
    out_code = DSA_BF16 if out.dtype == torch.bfloat16 else DSA_F32
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.dsa_sparse_mla(_p(q), _p(kv), _p(offsets), _p(indices), B, T, H, k, float(scale), kv_rows,
                              _p(out), out_code, _p(lse), _p(workspace), ws_bytes, _p(status),
                              _stream(stream)),
           "dsa_sparse_mla")


def sparse_mla_noalloc(q, kv, offsets, indices, B, T, H, k, scale, kv_rows, out, lse=None, status=None,
                       stream=None):
    """dsa_sparse_mla_noalloc: dsa_sparse_mla with the library's built-in scratch (no workspace)."""
    out_code = DSA_BF16 if out.dtype == torch.bfloat16 else DSA_F32
    _check(lib.dsa_sparse_mla_noalloc(_p(q), _p(kv), _p(offsets), _p(indices), B, T, H, k, float(scale), kv_rows,
                                      _p(out), out_code, _p(lse), _p(status), _stream(stream)),
           "dsa_sparse_mla_noalloc")


def cache_append(k_new, kv_new, offsets, B, T, k_cache, k_scale, kv_cache, kv_rows, status=None, stream=None):
    """dsa_cache_append: the newest T tokens' key (e4m3-quantised when the key
    cache is uint8) and latent rows into each sequence's last T cache rows."""
    code = DSA_E4M3 if (k_cache is not None and k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)) else DSA_BF16
    _check(lib.dsa_cache_append(_p(k_new), _p(kv_new), _p(offsets), B, T, code, _p(k_cache), _p(k_scale),
                                _p(kv_cache), kv_rows, _p(status), _stream(stream)), "dsa_cache_append")


def indexer_prestage(x, pos, rope_cos, rope_sin, y=None, status=None, stream=None):
    """dsa_indexer_prestage on x [n_rows, V, 128] bf16 (V vectors per row share
    pos[row]): rotary embedding of the rope half, then the Hadamard rotation,
    into y (a new tensor unless given; y may be x)."""
    if x.dim() != 3 or x.shape[-1] != 128:
        raise DSAError(1, "indexer_prestage: x must be [n_rows, V, 128]")
    if y is None:
        y = torch.empty_like(x)
    _check(lib.dsa_indexer_prestage(_p(x), _p(pos), x.shape[0], x.shape[1], _p(rope_cos), _p(rope_sin),
                                    rope_cos.shape[0], _p(y), _p(status), _stream(stream)), "dsa_indexer_prestage")
    return y


def quantize_queries(q_idx, w, n_rows, q_e4m3, w_out, stream=None):
    """dsa_quantize_queries: e4m3 codes of q_idx and w_out = w * q_scale."""
    _check(lib.dsa_quantize_queries(_p(q_idx), _p(w), n_rows, _p(q_e4m3), _p(w_out), _stream(stream)),
           "dsa_quantize_queries")


def _host_p(t: torch.Tensor):
    if t.is_cuda or not t.is_contiguous():
        raise DSAError(1, "host buffer must be a contiguous CPU tensor")
    return ctypes.c_void_p(t.data_ptr())


def copy_host_to_device(dst, src_host, stream=None):
    """dsa_copy_host_to_device: dst (CUDA) <- src_host (pinned CPU), by a kernel."""
    n = src_host.numel() * src_host.element_size()
    if dst.numel() * dst.element_size() != n:
        raise DSAError(1, "copy_host_to_device: sizes differ")
    _check(lib.dsa_copy_host_to_device(_p(dst), _host_p(src_host), n, _stream(stream)), "dsa_copy_host_to_device")


def copy_device_to_host(dst_host, src, stream=None):
    """dsa_copy_device_to_host: dst_host (pinned CPU) <- src (CUDA), by a kernel."""
    n = src.numel() * src.element_size()
    if dst_host.numel() * dst_host.element_size() != n:
        raise DSAError(1, "copy_device_to_host: sizes differ")
    _check(lib.dsa_copy_device_to_host(_host_p(dst_host), _p(src), n, _stream(stream)), "dsa_copy_device_to_host")


def debug_stall_attention(n_launches: int, wait_limit_ns: int = 0):
    """dsa_debug_stall_attention: the next n_launches attention launches take
    their timeout path after wait_limit_ns (a test hook)."""
    _check(lib.dsa_debug_stall_attention(n_launches, wait_limit_ns), "dsa_debug_stall_attention")


def decode_step_launches(B, max_end_pos, k, H) -> int:
    """Kernels one dsa_decode_step launches for these sizes."""
    return int(lib.dsa_decode_step_launches(B, max_end_pos, k, H))


def decode_step_workspace_size(B, max_end_pos, k, H) -> int:
    return int(lib.dsa_decode_step_workspace_size(B, max_end_pos, k, H))


def decode_step_workspace_layout(B, max_end_pos, k, H):
    """(scores byte offset, ld, indices byte offset, mla byte offset) inside the workspace."""
    so, ld, io, mo = ctypes.c_size_t(), ctypes.c_int64(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.dsa_decode_step_workspace_layout(B, max_end_pos, k, H, ctypes.byref(so), ctypes.byref(ld),
                                                ctypes.byref(io), ctypes.byref(mo)),
           "dsa_decode_step_workspace_layout")
    return so.value, ld.value, io.value, mo.value


def decode_step(q_idx, w, k_idx, k_scale, q, kv, offsets, B, max_end_pos, kv_rows, k, H, scale, out,
                lse=None, workspace=None, status=None, stream=None):
    """dsa_decode_step: indexer -> top-k -> sparse MLA for T=1 queries."""
    out_code = DSA_BF16 if out.dtype == torch.bfloat16 else DSA_F32
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.dsa_decode_step(_p(q_idx), _p(w), _p(k_idx), _p(k_scale), _dtype_code(q_idx), _p(q), _p(kv),
                               _p(offsets), B, max_end_pos, kv_rows, k, H, float(scale), _p(out), out_code,
                               _p(lse), _p(workspace), ws_bytes, _p(status), _stream(stream)),
           "dsa_decode_step")
