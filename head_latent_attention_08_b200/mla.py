"""Thin Python binding of libmla_b200.so (ctypes). Argument marshalling only: every step runs in
the library's CUDA kernels. Torch tensors supply device memory and the current CUDA stream.

The functions carry the C names (``mla_append_latent``, ``mla_absorb_weights``,
``mla_decode_absorbed``, ``mla_out_project``, ``mla_linear`` ...). A non-zero status raises
:class:`MLAError`. ``decode_step`` and ``gated_mla`` chain those calls for the two workloads.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_b200.so")

MLA_OK = 0
MLA_F32, MLA_BF16, MLA_FP8_E4M3 = 0, 1, 2
MLA_ABSORB_QUERY, MLA_FOLD_QK, MLA_FOLD_VO = 0, 1, 2
MLA_APPEND_NORM, MLA_APPEND_ROPE = 1, 2
MLA_DECODE_CAUSAL, MLA_DECODE_OUT_BF16 = 1, 2
MLA_LINEAR_SIGMOID, MLA_LINEAR_W_KN = 1, 2
MLA_ERR_SHAPE, MLA_ERR_TIMEOUT = 2, 7
MLA_IO_DEVICE, MLA_IO_HOST = 0, 1

EXPORTED = (
    "mla_status_string", "mla_abi_version", "mla_append_latent", "mla_absorb_weights",
    "mla_decode_workspace_size", "mla_decode_absorbed", "mla_out_project_workspace_size",
    "mla_out_project", "mla_linear", "mla_check_status", "mla_set_wait_limit", "mla_launch_count",
    "mla_set_decode_clusters", "mla_wait_selftest", "mla_decode_absorbed_noalloc",
    "mla_project_workspace_size", "mla_project_inputs", "mla_decode_step_workspace_size", "mla_decode_step",
    "mla_lse_merge", "mla_prefill_attention", "mla_append_latent_fp8", "mla_decode_absorbed_fp8",
    "mla_out_project_bf16",
)


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class mla_dims(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("kv_lora_rank", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("qk_nope", ctypes.c_int32),
                ("v_head", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("kq_scale", ctypes.c_float)]


def dims(n_heads, kv_lora_rank, rope_dim=0, qk_nope=0, v_head=0, d_model=0, kq_scale=0.0):
    return mla_dims(n_heads, kv_lora_rank, rope_dim, qk_nope, v_head, d_model, kq_scale)


class mla_step_weights(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in ("w_cq", "w_qc", "w_qr", "w_dkv", "w_uk", "w_uv", "w_o")]


_lib: Optional[ctypes.CDLL] = None

_P, _I32, _I64, _U32, _F, _SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                 ctypes.c_float, ctypes.c_size_t)
_DIMS = ctypes.POINTER(mla_dims)
_SIGS = {
    "mla_status_string": (ctypes.c_char_p, [_I32]),
    "mla_abi_version": (_I32, []),
    "mla_append_latent": (_I32, [_DIMS, _I32, _P, _I64, _P, _P, _P, _P, _I64, _U32, _F, _F, _P]),
    "mla_absorb_weights": (_I32, [_DIMS, _I32, _I32, _P, _P, _P, _I64, _P, _P]),
    "mla_decode_workspace_size": (_I32, [_DIMS, _I32, _I32, _I32, _I64, _I64, _U32, ctypes.POINTER(_SZ)]),
    "mla_decode_absorbed": (_I32, [_DIMS, _I32, _P, _P, _P, _I32, _I32, _I64, _I64, _U32, _P, _P, _P,
                                   _SZ, _P]),
    "mla_out_project_workspace_size": (_I32, [_DIMS, _I32, _I64, ctypes.POINTER(_SZ)]),
    "mla_out_project": (_I32, [_DIMS, _I32, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "mla_out_project_bf16": (_I32, [_DIMS, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "mla_linear": (_I32, [_I32, _P, _P, _I64, _I64, _I64, _U32, _P, _P]),
    "mla_check_status": (_I32, [_P, ctypes.POINTER(_I32)]),
    "mla_set_wait_limit": (_I32, [_I64]),
    "mla_launch_count": (_I64, []),
    "mla_set_decode_clusters": (_I32, [_I32]),
    "mla_wait_selftest": (_I32, [_P]),
    "mla_decode_absorbed_noalloc": (_I32, [_DIMS, _I32, _P, _P, _P, _I32, _I32, _I64, _I64, _U32, _P, _P,
                                           _P]),
    "mla_project_workspace_size": (_I32, [_DIMS, _I32, _I32, _I64, ctypes.POINTER(_SZ)]),
    "mla_project_inputs": (_I32, [_DIMS, _I32, _I32, _P, _P, _P, _P, _P, _I64, _P, _P, _P, _P, _I64, _P, _U32,
                                  _F, _F, _P, _SZ, _P]),
    "mla_decode_step_workspace_size": (_I32, [_DIMS, _I32, _I32, _I32, _I64, _I64, ctypes.POINTER(_SZ)]),
    "mla_decode_step": (_I32, [_DIMS, _I32, _I32, ctypes.POINTER(mla_step_weights), _P, _P, _P, _I32, _I64,
                               _I64, _P, _P, _U32, _F, _F, _P, _I32, _P, _SZ, _P]),
    "mla_lse_merge": (_I32, [_DIMS, _I32, ctypes.POINTER(_P), ctypes.POINTER(_P), _I64, _I64, _P, _P, _P]),
    "mla_prefill_attention": (_I32, [_I32, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _F, _U32, _P, _P]),
    "mla_append_latent_fp8": (_I32, [_DIMS, _P, _I64, _P, _P, _P, _P, _I64, _U32, _F, _F, _F, _P]),
    "mla_decode_absorbed_fp8": (_I32, [_DIMS, _I32, _P, _P, _F, _P, _I32, _I32, _I64, _I64, _U32, _P, _P, _P, _SZ,
                                       _P]),
}


def lib() -> ctypes.CDLL:
    """Open the library (once). Raises if it is missing: there is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m head_latent_attention_08_b200.build` (nvcc, sm_100a)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().mla_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - only when the library itself cannot load
        return f"status {status}"


def _check(status: int, where: str):
    if status != MLA_OK:
        raise MLAError(status, where)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return MLA_F32
    if t == torch.bfloat16:
        return MLA_BF16
    if t in (torch.uint8, torch.float8_e4m3fn):
        return MLA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _host_ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("this argument is host memory")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


# --------------------------------------------------------------------------------------------
# the C entry points
# --------------------------------------------------------------------------------------------

def mla_append_latent(d: mla_dims, cache: torch.Tensor, row_idx: torch.Tensor, c_new: torch.Tensor,
                      kpe_new: Optional[torch.Tensor], positions: Optional[torch.Tensor], flags: int,
                      eps: float = 1e-6, rope_theta: float = 10000.0, stream=None) -> None:
    assert row_idx.dtype == torch.int64 and c_new.dtype == torch.float32
    assert kpe_new is None or kpe_new.dtype == torch.float32
    assert positions is None or positions.dtype == torch.int32
    n_new = row_idx.numel()
    _check(lib().mla_append_latent(ctypes.byref(d), _dtype_code(cache.dtype), _ptr(cache), cache.shape[0],
                                   _ptr(row_idx), _ptr(c_new), _ptr(kpe_new), _ptr(positions), n_new,
                                   flags, eps, rope_theta, _stream(stream)), "mla_append_latent")


def mla_absorb_weights(d: mla_dims, mode: int, x: torch.Tensor, x_pe: Optional[torch.Tensor],
                       w: torch.Tensor, n_rows: int, out: torch.Tensor, stream=None) -> None:
    _check(lib().mla_absorb_weights(ctypes.byref(d), _dtype_code(x.dtype), mode, _ptr(x), _ptr(x_pe),
                                    _ptr(w), n_rows, _ptr(out), _stream(stream)), "mla_absorb_weights")


def mla_decode_workspace_size(d: mla_dims, dtype: torch.dtype, batch: int, n_q: int, max_seqlen: int,
                              total_rows: int, flags: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mla_decode_workspace_size(ctypes.byref(d), _dtype_code(dtype), batch, n_q, max_seqlen,
                                           total_rows, flags, ctypes.byref(n)),
           "mla_decode_workspace_size")
    return int(n.value)


def mla_decode_absorbed(d: mla_dims, q_abs: torch.Tensor, cache: torch.Tensor, cu_seqlens: torch.Tensor,
                        batch: int, n_q: int, max_seqlen: int, flags: int, out_lat: torch.Tensor,
                        lse: Optional[torch.Tensor], workspace: Optional[torch.Tensor],
                        stream=None) -> None:
    assert cu_seqlens.dtype == torch.int32
    assert out_lat.dtype == (torch.bfloat16 if flags & MLA_DECODE_OUT_BF16 else torch.float32)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().mla_decode_absorbed(ctypes.byref(d), _dtype_code(q_abs.dtype), _ptr(q_abs), _ptr(cache),
                                     _ptr(cu_seqlens), batch, n_q, max_seqlen, cache.shape[0], flags,
                                     _ptr(out_lat), _ptr(lse), _ptr(workspace), ws_bytes,
                                     _stream(stream)), "mla_decode_absorbed")


MLA_DECODE_NOALLOC_MAX_BYTES = 40 << 20


def mla_decode_absorbed_noalloc(d: mla_dims, q_abs: torch.Tensor, cache: torch.Tensor,
                                cu_seqlens: torch.Tensor, batch: int, n_q: int, max_seqlen: int, flags: int,
                                out_lat: torch.Tensor, lse: Optional[torch.Tensor], stream=None) -> None:
    assert cu_seqlens.dtype == torch.int32
    assert out_lat.dtype == (torch.bfloat16 if flags & MLA_DECODE_OUT_BF16 else torch.float32)
    _check(lib().mla_decode_absorbed_noalloc(ctypes.byref(d), _dtype_code(q_abs.dtype), _ptr(q_abs),
                                             _ptr(cache), _ptr(cu_seqlens), batch, n_q, max_seqlen,
                                             cache.shape[0], flags, _ptr(out_lat), _ptr(lse),
                                             _stream(stream)), "mla_decode_absorbed_noalloc")


def mla_out_project_workspace_size(d: mla_dims, dtype: torch.dtype, n_rows: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mla_out_project_workspace_size(ctypes.byref(d), _dtype_code(dtype), n_rows,
                                                ctypes.byref(n)), "mla_out_project_workspace_size")
    return int(n.value)


def mla_out_project(d: mla_dims, out_lat: torch.Tensor, w_uv: torch.Tensor, w_o: torch.Tensor,
                    gate: Optional[torch.Tensor], n_rows: int, y: torch.Tensor,
                    workspace: torch.Tensor, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().mla_out_project(ctypes.byref(d), _dtype_code(w_uv.dtype), _ptr(out_lat), _ptr(w_uv),
                                 _ptr(w_o), _ptr(gate), n_rows, _ptr(y), _ptr(workspace), ws_bytes,
                                 _stream(stream)), "mla_out_project")


def mla_out_project_bf16(d: mla_dims, out_lat: torch.Tensor, w_uv: torch.Tensor, w_o: torch.Tensor,
                         gate: Optional[torch.Tensor], n_rows: int, y: torch.Tensor,
                         workspace: torch.Tensor, stream=None) -> None:
    """mla_out_project with a bf16 out_lat (the decode's MLA_DECODE_OUT_BF16 output)."""
    assert out_lat.dtype == torch.bfloat16
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().mla_out_project_bf16(ctypes.byref(d), _ptr(out_lat), _ptr(w_uv), _ptr(w_o), _ptr(gate), n_rows,
                                      _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)), "mla_out_project_bf16")


def mla_linear(x: torch.Tensor, w: torch.Tensor, m: int, n: int, k: int, flags: int, y: torch.Tensor,
               stream=None) -> None:
    _check(lib().mla_linear(_dtype_code(x.dtype), _ptr(x), _ptr(w), m, n, k, flags, _ptr(y),
                            _stream(stream)), "mla_linear")


def mla_project_workspace_size(d: mla_dims, dtype: torch.dtype, q_rank: int, n_rows: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mla_project_workspace_size(ctypes.byref(d), _dtype_code(dtype), q_rank, n_rows, ctypes.byref(n)),
           "mla_project_workspace_size")
    return int(n.value)


def mla_project_inputs(d: mla_dims, q_rank: int, x: torch.Tensor, w_cq: torch.Tensor, w_qc: torch.Tensor,
                       w_qr: Optional[torch.Tensor], w_dkv: torch.Tensor, positions: Optional[torch.Tensor],
                       q_nope: torch.Tensor, q_pe: Optional[torch.Tensor], cache: torch.Tensor,
                       row_idx: torch.Tensor, flags: int, workspace: torch.Tensor, eps: float = 1e-6,
                       rope_theta: float = 10000.0, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().mla_project_inputs(ctypes.byref(d), _dtype_code(x.dtype), q_rank, _ptr(x), _ptr(w_cq), _ptr(w_qc),
                                    _ptr(w_qr), _ptr(w_dkv), x.shape[0], _ptr(positions), _ptr(q_nope),
                                    _ptr(q_pe), _ptr(cache), cache.shape[0], _ptr(row_idx), flags, eps,
                                    rope_theta, _ptr(workspace), ws_bytes, _stream(stream)),
           "mla_project_inputs")


def mla_decode_step_workspace_size(d: mla_dims, dtype: torch.dtype, q_rank: int, batch: int, max_seqlen: int,
                                   total_rows: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mla_decode_step_workspace_size(ctypes.byref(d), _dtype_code(dtype), q_rank, batch, max_seqlen,
                                                total_rows, ctypes.byref(n)), "mla_decode_step_workspace_size")
    return int(n.value)


def mla_decode_step(d: mla_dims, q_rank: int, w: mla_step_weights, x: torch.Tensor, cache: torch.Tensor,
                    cu_seqlens: torch.Tensor, batch: int, max_seqlen: int, row_idx: torch.Tensor,
                    positions: Optional[torch.Tensor], flags: int, y: torch.Tensor, io: int,
                    workspace: torch.Tensor, eps: float = 1e-6, rope_theta: float = 10000.0, stream=None) -> None:
    """One decode step through the C ABI. With io == MLA_IO_HOST, x, y, cu_seqlens, row_idx and
    positions are host tensors (page-locked for asynchronous copies)."""
    p = _host_ptr if io == MLA_IO_HOST else _ptr
    assert cu_seqlens.dtype == torch.int32 and row_idx.dtype == torch.int64
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().mla_decode_step(ctypes.byref(d), _dtype_code(cache.dtype), q_rank, ctypes.byref(w), p(x),
                                 _ptr(cache), p(cu_seqlens), batch, max_seqlen, cache.shape[0], p(row_idx),
                                 p(positions), flags, eps, rope_theta, p(y), io, _ptr(workspace), ws_bytes,
                                 _stream(stream)), "mla_decode_step")


MLA_MERGE_MAX_PARTS = 16


def mla_lse_merge(d: mla_dims, out_lat_parts, lse_parts, row_begin: int, n_rows: int, out_lat: torch.Tensor,
                  lse: Optional[torch.Tensor], stream=None) -> None:
    """Merge partial decode results by their log-sum-exp. The parts are device tensors or raw device
    addresses (e.g. peers' symmetric-memory buffers)."""
    def addr(x):
        return x if isinstance(x, int) else _ptr(x)
    n = len(out_lat_parts)
    if len(lse_parts) != n:
        raise ValueError("one lse part per out_lat part")
    po = (_P * n)(*[addr(x) for x in out_lat_parts])
    pl = (_P * n)(*[addr(x) for x in lse_parts])
    _check(lib().mla_lse_merge(ctypes.byref(d), n, po, pl, row_begin, n_rows, _ptr(out_lat), _ptr(lse),
                               _stream(stream)), "mla_lse_merge")


def mla_prefill_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: Optional[torch.Tensor],
                          batch: int, seq: int, n_heads: int, head_dim: int, scale: float, flags: int,
                          out: torch.Tensor, stream=None) -> None:
    _check(lib().mla_prefill_attention(_dtype_code(q.dtype), _ptr(q), _ptr(k), _ptr(v), _ptr(gate), batch, seq,
                                       n_heads, head_dim, scale, flags, _ptr(out), _stream(stream)),
           "mla_prefill_attention")


def mla_append_latent_fp8(d: mla_dims, cache: torch.Tensor, row_idx: torch.Tensor, c_new: torch.Tensor,
                          kpe_new: Optional[torch.Tensor], positions: Optional[torch.Tensor], flags: int,
                          cache_scale: float = 1.0, eps: float = 1e-6, rope_theta: float = 10000.0,
                          stream=None) -> None:
    """cache: a uint8 (or float8_e4m3fn) tensor [rows, d_c + d_r] holding e4m3 codes."""
    _check(lib().mla_append_latent_fp8(ctypes.byref(d), _ptr(cache), cache.shape[0], _ptr(row_idx), _ptr(c_new),
                                       _ptr(kpe_new), _ptr(positions), row_idx.numel(), flags, eps, rope_theta,
                                       cache_scale, _stream(stream)), "mla_append_latent_fp8")


def mla_decode_absorbed_fp8(d: mla_dims, q_abs: torch.Tensor, cache: torch.Tensor, cache_scale: float,
                            cu_seqlens: torch.Tensor, batch: int, n_q: int, max_seqlen: int, flags: int,
                            out_lat: torch.Tensor, lse: Optional[torch.Tensor], workspace: Optional[torch.Tensor],
                            stream=None) -> None:
    assert cu_seqlens.dtype == torch.int32
    assert out_lat.dtype == (torch.bfloat16 if flags & MLA_DECODE_OUT_BF16 else torch.float32)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().mla_decode_absorbed_fp8(ctypes.byref(d), _dtype_code(q_abs.dtype), _ptr(q_abs), _ptr(cache),
                                         cache_scale, _ptr(cu_seqlens), batch, n_q, max_seqlen, cache.shape[0],
                                         flags, _ptr(out_lat), _ptr(lse), _ptr(workspace), ws_bytes,
                                         _stream(stream)), "mla_decode_absorbed_fp8")


def mla_check_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().mla_check_status(_stream(stream), ctypes.byref(v)), "mla_check_status")
    return int(v.value)


def mla_launch_count() -> int:
    return int(lib().mla_launch_count())


def mla_set_decode_clusters(n: int) -> None:
    _check(lib().mla_set_decode_clusters(int(n)), "mla_set_decode_clusters")


def mla_set_wait_limit(limit_ns: int) -> None:
    _check(lib().mla_set_wait_limit(int(limit_ns)), "mla_set_wait_limit")


def mla_wait_selftest(stream=None) -> None:
    _check(lib().mla_wait_selftest(_stream(stream)), "mla_wait_selftest")


# --------------------------------------------------------------------------------------------
# chained calls
# --------------------------------------------------------------------------------------------

def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned scratch buffer of at least ``nbytes`` bytes (caller-owned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class DecodeStep:
    """One absorbed-decode step over resident weights and cache: append the new tokens' latents,
    absorb the queries, attend over the latent cache, project. Buffers are allocated once here;
    ``__call__`` only launches the library's kernels."""

    def __init__(self, d: mla_dims, dtype: torch.dtype, batch: int, n_q: int, max_seqlen: int,
                 cache: torch.Tensor, cu_seqlens: torch.Tensor, w_uk: torch.Tensor,
                 w_uv: torch.Tensor, w_o: torch.Tensor, causal: bool = True,
                 append_flags: int = MLA_APPEND_NORM | MLA_APPEND_ROPE):
        dev = cache.device
        self.d, self.dtype, self.batch, self.n_q, self.max_seqlen = d, dtype, batch, n_q, max_seqlen
        self.cache, self.cu, self.w_uk, self.w_uv, self.w_o = cache, cu_seqlens, w_uk, w_uv, w_o
        self.flags = MLA_DECODE_CAUSAL if causal else 0
        self.append_flags = append_flags
        nq = batch * n_q
        H, W = d.n_heads, d.kv_lora_rank + d.rope_dim
        self.q_abs = torch.empty(nq, H, W, dtype=dtype, device=dev)
        self.out_lat = torch.empty(nq, H, d.kv_lora_rank, dtype=torch.float32, device=dev)
        self.lse = torch.empty(nq, H, dtype=torch.float32, device=dev)
        self.y = torch.empty(nq, d.d_model, dtype=dtype, device=dev)
        self.ws_dec = workspace(mla_decode_workspace_size(d, dtype, batch, n_q, max_seqlen,
                                                          cache.shape[0], self.flags), dev)
        self.ws_out = workspace(mla_out_project_workspace_size(d, dtype, nq), dev)

    def __call__(self, q_nope, q_pe, c_new, kpe_new, row_idx, positions, stream=None, y=None):
        d = self.d
        nq = self.batch * self.n_q
        y = self.y if y is None else y
        mla_append_latent(d, self.cache, row_idx, c_new, kpe_new, positions, self.append_flags,
                          stream=stream)
        mla_absorb_weights(d, MLA_ABSORB_QUERY, q_nope, q_pe if d.rope_dim else None, self.w_uk, nq,
                           self.q_abs, stream=stream)
        mla_decode_absorbed(d, self.q_abs, self.cache, self.cu, self.batch, self.n_q, self.max_seqlen,
                            self.flags, self.out_lat, self.lse, self.ws_dec, stream=stream)
        mla_out_project(d, self.out_lat, self.w_uv, self.w_o, None, nq, y, self.ws_out,
                        stream=stream)
        return y


class DecodeLayerStep:
    """One decode step of the attention layer from hidden states to outputs through the library's
    single step call (mla_decode_step): input projections with the append, query absorption,
    decode over the latent cache, value and output projection. One new token per sequence."""

    def __init__(self, d: mla_dims, q_rank: int, batch: int, max_seqlen: int, cache: torch.Tensor,
                 cu_seqlens: torch.Tensor, w_cq, w_qc, w_qr, w_dkv, w_uk, w_uv, w_o,
                 append_flags: int = MLA_APPEND_NORM | MLA_APPEND_ROPE):
        self.d, self.q_rank, self.batch, self.max_seqlen = d, q_rank, batch, max_seqlen
        self.cache, self.cu, self.append_flags = cache, cu_seqlens, append_flags
        self.tensors = (w_cq, w_qc, w_qr, w_dkv, w_uk, w_uv, w_o)     # kept alive with the struct
        self.w = mla_step_weights(*[None if t is None else _ptr(t) for t in self.tensors])
        self.y = torch.empty(batch, d.d_model, dtype=cache.dtype, device=cache.device)
        self.ws = workspace(mla_decode_step_workspace_size(d, cache.dtype, q_rank, batch, max_seqlen,
                                                           cache.shape[0]), cache.device)

    def __call__(self, x, row_idx, positions, y=None, io: int = MLA_IO_DEVICE, cu_seqlens=None, stream=None):
        """Device io: every tensor on the GPU. Host io: x, y, row_idx, positions and cu_seqlens
        (defaulting to the step's, copied to the host once) are host tensors."""
        y = self.y if y is None else y
        cu = self.cu if cu_seqlens is None else cu_seqlens
        if io == MLA_IO_HOST and cu.is_cuda:
            self.cu_host = getattr(self, "cu_host", None)
            if self.cu_host is None:
                self.cu_host = cu.cpu().pin_memory()
            cu = self.cu_host
        mla_decode_step(self.d, self.q_rank, self.w, x, self.cache, cu, self.batch, self.max_seqlen, row_idx,
                        positions, self.append_flags, y, io, self.ws, stream=stream)
        return y


class HostStream:
    """Decode steps fed from pinned host memory, with the transfers overlapped with the compute.
    While step k runs on the compute stream, step k+1's inputs travel host -> device on one side
    stream and step k-1's output travels device -> host on another. Two sets of device buffers
    alternate, and events order every reuse: a buffer set takes new inputs once the step that read
    it is done, and its output buffer is written again once its previous output has reached the
    host. ``submit`` enqueues one step and returns at once; ``wait(stream)`` makes ``stream`` wait
    for every submitted step's output to be in host memory."""

    def __init__(self, step: DecodeStep, stream=None):
        self.step = step
        dev = step.cache.device
        self.compute = stream if stream is not None else torch.cuda.current_stream(dev)
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        d, nq = step.d, step.batch * step.n_q

        def buffers():
            return dict(q_nope=torch.empty(nq, d.n_heads, d.qk_nope, dtype=step.dtype, device=dev),
                        q_pe=torch.empty(nq, d.n_heads, d.rope_dim, dtype=step.dtype, device=dev),
                        c_new=torch.empty(nq, d.kv_lora_rank, dtype=torch.float32, device=dev),
                        kpe_new=torch.empty(nq, d.rope_dim, dtype=torch.float32, device=dev),
                        y=torch.empty_like(step.y))

        self.buf = [buffers(), buffers()]
        self.inputs_in = [torch.cuda.Event() for _ in range(2)]
        self.step_done = [torch.cuda.Event() for _ in range(2)]
        self.output_out = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]
        self.k = 0

    def submit(self, h_q_nope, h_q_pe, h_c_new, h_kpe, row_idx, positions, h_y):
        i = self.k & 1
        b = self.buf[i]
        with torch.cuda.stream(self.h2d):
            if self.used[i]:
                self.h2d.wait_event(self.step_done[i])
            b["q_nope"].copy_(h_q_nope, non_blocking=True)
            b["q_pe"].copy_(h_q_pe, non_blocking=True)
            b["c_new"].copy_(h_c_new, non_blocking=True)
            b["kpe_new"].copy_(h_kpe, non_blocking=True)
            self.inputs_in[i].record(self.h2d)
        self.compute.wait_event(self.inputs_in[i])
        if self.used[i]:
            self.compute.wait_event(self.output_out[i])
        with torch.cuda.stream(self.compute):
            self.step(b["q_nope"], b["q_pe"], b["c_new"], b["kpe_new"], row_idx, positions,
                      stream=self.compute, y=b["y"])
            self.step_done[i].record(self.compute)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.step_done[i])
            h_y.copy_(b["y"], non_blocking=True)
            self.output_out[i].record(self.d2h)
        self.used[i] = True
        self.k += 1

    def wait(self, stream=None):
        s = stream if stream is not None else self.compute
        for i in range(2):
            if self.used[i]:
                s.wait_event(self.output_out[i])


def gated_mla(x: torch.Tensor, wq: torch.Tensor, wc: torch.Tensor, wk: torch.Tensor, wv: torch.Tensor,
              wg: torch.Tensor, wo: torch.Tensor, num_heads: int, causal: bool = True, stream=None,
              route: str = "auto"):
    """Gated MLA prefill. Q, C and sigmoid(X Wg^T) come from mla_linear; then either
    * route "unabsorbed": K = C Wk^T and V = C Wv^T by mla_linear, attention of the D_h-wide heads with
      the gate by mla_prefill_attention, Y = O Wo^T by mla_linear; or
    * route "absorbed": the query absorbed into the latent per head (W_UK[h] = rows h*D_h.. of Wk),
      attention over the latent C, then W_UV[h] = rows of Wv, the gate and Wo by mla_out_project.
    "auto" takes the un-absorbed route where its tensor-core kernel applies (bf16, D_h = 128). Returns
    {"output": [B, S, D], "latent_cache": [B, S, L]}; the inputs are not modified."""
    B, S, D = x.shape
    L = wc.shape[0]
    H = num_heads
    if D % H:
        raise ValueError("model width must be divisible by the head count")
    Dh = D // H
    dev, dt = x.device, x.dtype
    if route == "auto":
        route = "unabsorbed" if (dt == torch.bfloat16 and Dh == 128) else "absorbed"
    if route not in ("absorbed", "unabsorbed"):
        raise ValueError("route is 'auto', 'absorbed' or 'unabsorbed'")
    x2 = x.reshape(B * S, D)
    q = torch.empty(B * S, D, dtype=dt, device=dev)
    c = torch.empty(B * S, L, dtype=dt, device=dev)
    g = torch.empty(B * S, D, dtype=dt, device=dev)
    mla_linear(x2, wq, B * S, D, D, 0, q, stream)
    mla_linear(x2, wc, B * S, L, D, 0, c, stream)
    mla_linear(x2, wg, B * S, D, D, MLA_LINEAR_SIGMOID, g, stream)
    if route == "unabsorbed":
        k = torch.empty(B * S, D, dtype=dt, device=dev)
        v = torch.empty(B * S, D, dtype=dt, device=dev)
        mla_linear(c, wk, B * S, D, L, 0, k, stream)
        mla_linear(c, wv, B * S, D, L, 0, v, stream)
        o = torch.empty(B * S, D, dtype=dt, device=dev)
        mla_prefill_attention(q, k, v, g, B, S, H, Dh, 1.0 / math.sqrt(Dh), MLA_DECODE_CAUSAL if causal else 0, o,
                              stream)
        y = torch.empty(B * S, D, dtype=dt, device=dev)
        mla_linear(o, wo, B * S, D, D, 0, y, stream)
        return {"output": y.reshape(B, S, D), "latent_cache": c.reshape(B, S, L)}
    d = dims(H, L, 0, Dh, Dh, D, 1.0 / math.sqrt(Dh))
    q_abs = torch.empty(B * S, H, L, dtype=dt, device=dev)
    mla_absorb_weights(d, MLA_ABSORB_QUERY, q, None, wk, B * S, q_abs, stream)
    cu = torch.arange(0, (B + 1) * S, S, dtype=torch.int32, device=dev)
    flags = MLA_DECODE_CAUSAL if causal else 0
    out_lat = torch.empty(B * S, H, L, dtype=torch.float32, device=dev)
    ws = workspace(mla_decode_workspace_size(d, dt, B, S, S, B * S, flags), dev)
    mla_decode_absorbed(d, q_abs, c, cu, B, S, S, flags, out_lat, None, ws, stream)
    y = torch.empty(B * S, D, dtype=dt, device=dev)
    ws2 = workspace(mla_out_project_workspace_size(d, dt, B * S), dev)
    mla_out_project(d, out_lat, wv, wo, g, B * S, y, ws2, stream)
    return {"output": y.reshape(B, S, D), "latent_cache": c.reshape(B, S, L)}
