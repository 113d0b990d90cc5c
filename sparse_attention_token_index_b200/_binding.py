"""ctypes binding of ``libdsa_index.so`` (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np
import torch

DSA_DTYPE_BF16 = 0
DSA_DTYPE_FP32 = 1
DSA_DTYPE_FP8_E4M3 = 2
DSA_GROUP_REFINE = 0
DSA_GROUP_REUSE = 1
DSA_GROUP_REFINE_LOCAL = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
# DSA_LIB overrides the in-tree library (to compare builds)
lib_path = os.environ.get("DSA_LIB") or os.path.join(_HERE, "libdsa_index.so")

EXPORTED_SYMBOLS = (
    "dsa_status_string", "dsa_version", "dsa_check_status", "dsa_debug_set_wait",
    "dsa_index_dense_workspace_size", "dsa_index_dense",
    "dsa_index_group_workspace_size", "dsa_index_group",
    "dsa_index_decode_workspace_size", "dsa_index_decode",
    "dsa_debug_scores", "dsa_index_dense_static",
    "dsa_kernel_timer_start", "dsa_kernel_timer_stop",
    "dsa_index_decode_group_workspace_size", "dsa_index_decode_group",
    "dsa_index_block_routed_workspace_size", "dsa_index_block_routed",
    "dsa_ivf_index_size", "dsa_ivf_build_workspace_size", "dsa_ivf_build",
    "dsa_index_ivf_routed_workspace_size", "dsa_index_ivf_routed",
    "dsa_index_dense_host_staging_size", "dsa_index_dense_host",
    "dsa_index_group_host_staging_size", "dsa_index_group_host",
    "dsa_index_decode_host_staging_size", "dsa_index_decode_host",
)


class DsaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = _status_text(status) if _LIB is not None else str(status)
        super().__init__(f"{what}: {msg} ({status})" if what else f"{msg} ({status})")


_LIB = None

_c_int, _c_i64, _c_sz, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
_SIGS = {
    "dsa_status_string": (ctypes.c_char_p, [_c_int]),
    "dsa_version": (_c_int, []),
    "dsa_debug_set_wait": (_c_int, [ctypes.c_uint, _c_int]),
    "dsa_check_status": (_c_int, [_vp, _vp]),
    "dsa_index_dense_workspace_size": (_c_int, [_c_int] * 7 + [ctypes.POINTER(_c_sz)]),
    "dsa_index_dense": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                 _c_int, _vp, _vp, _vp, _c_sz, _vp]),
    "dsa_index_group_workspace_size": (_c_int, [_c_int] * 9 + [ctypes.POINTER(_c_sz)]),
    "dsa_index_group": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                 _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_sz, _vp]),
    "dsa_index_decode_workspace_size": (_c_int, [_c_int] * 8 + [ctypes.POINTER(_c_sz)]),
    "dsa_index_decode": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int,
                                  _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_sz, _vp]),
    "dsa_debug_scores": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                  _vp, _vp, _c_sz, _vp]),
    "dsa_index_dense_static": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _vp, _vp,
                                        _vp]),
    "dsa_kernel_timer_start": (_c_int, [_c_int]),
    "dsa_index_decode_group_workspace_size": (_c_int, [_c_int] * 9 + [ctypes.POINTER(_c_sz)]),
    "dsa_index_block_routed_workspace_size": (_c_int, [_c_int] * 8 + [ctypes.POINTER(_c_sz)]),
    "dsa_ivf_index_size": (_c_int, [_c_int] * 3 + [ctypes.POINTER(_c_sz)]),
    "dsa_ivf_build_workspace_size": (_c_int, [_c_int] * 6 + [ctypes.POINTER(_c_sz)]),
    "dsa_ivf_build": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_sz, _vp,
                               _c_sz, _vp]),
    "dsa_index_ivf_routed_workspace_size": (_c_int, [_c_int] * 10 + [ctypes.POINTER(_c_sz)]),
    "dsa_index_ivf_routed": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                      _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_sz, _vp]),
    "dsa_index_block_routed": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                        _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_sz, _vp]),
    "dsa_index_decode_group": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int,
                                        _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _c_sz, _vp]),
    "dsa_kernel_timer_stop": (_c_int, [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_c_int)]),
    "dsa_index_dense_host_staging_size": (_c_int, [_c_int] * 7 + [ctypes.POINTER(_c_sz)]),
    "dsa_index_dense_host": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                      _c_int, _c_int, _vp, _vp, _vp, _c_sz, _vp]),
    "dsa_index_group_host_staging_size": (_c_int, [_c_int] * 10 + [ctypes.POINTER(_c_sz)]),
    "dsa_index_group_host": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                      _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_sz, _vp]),
    "dsa_index_decode_host_staging_size": (_c_int, [_c_int, _c_int, _c_i64] + [_c_int] * 6
                                           + [ctypes.POINTER(_c_sz)]),
    "dsa_index_decode_host": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int,
                                       _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_sz, _vp]),
}


def lib():
    """The loaded library; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(f"{lib_path} is missing: build it with "
                               "`python -m sparse_attention_token_index_b200.build`")
        L = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def _status_text(s: int) -> str:
    return lib().dsa_status_string(int(s)).decode()


def _check(status: int, what: str):
    if status != 0:
        raise DsaError(status, what)


def _dtype_code(t: torch.Tensor, allow_fp8=False) -> int:
    if t.dtype == torch.bfloat16:
        return DSA_DTYPE_BF16
    if t.dtype == torch.float32:
        return DSA_DTYPE_FP32
    if allow_fp8 and t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_DTYPE_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check_shapes(Q=None, w=None, K=None, K_scale=None, n_keys=None):
    """Shapes the library relies on but cannot see through its pointers: a
    mismatch would make it read past a buffer.  Q [T, H, d]; w float32
    [T, H]; K [N, d]; K_scale float32 [N] (N = K's rows, or n_keys)."""
    d = None
    if Q is not None:
        if Q.dim() != 3:
            raise ValueError("Q must be [T, H, d]")
        T, H, d = Q.shape
        if w is None or w.dtype != torch.float32 or tuple(w.shape) != (T, H):
            raise ValueError(f"w must be float32 [{T}, {H}]")
    if K is not None:
        if K.dim() != 2 or (d is not None and K.shape[1] != d):
            raise ValueError(f"K must be [N, {d if d is not None else 'd'}]")
        n_keys = K.shape[0]
    if K_scale is not None:
        if K_scale.dtype != torch.float32 or tuple(K_scale.shape) != (n_keys,):
            raise ValueError(f"K_scale must be float32 [{n_keys}]")


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (the indexer has no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _workspace(nbytes: int, device, workspace):
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace has {workspace.numel()} bytes, needs {nbytes}")
        return workspace
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def dense_workspace_bytes(T, N, H, d, k, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_dense_workspace_size(T, N, H, d, k, q_dtype, k_dtype, ctypes.byref(n)),
           "dsa_index_dense_workspace_size")
    return n.value


def group_workspace_bytes(T, N, H, d, k, group, bank, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_group_workspace_size(T, N, H, d, k, group, bank, q_dtype, k_dtype, ctypes.byref(n)),
           "dsa_index_group_workspace_size")
    return n.value


def decode_workspace_bytes(B, total_q, max_keys, H, d, k, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_decode_workspace_size(B, total_q, max_keys, H, d, k, q_dtype, k_dtype,
                                                 ctypes.byref(n)), "dsa_index_decode_workspace_size")
    return n.value


def dsa_check_status(workspace: torch.Tensor, stream=None) -> None:
    """Waits for the stream and raises if a kernel recorded a device-side failure."""
    _check(lib().dsa_check_status(_ptr(workspace), _stream(stream)), "device status")


def dsa_debug_set_wait(budget_us: int = 0, hold_first_tile: bool = False) -> None:
    """Failure-path control for tests: the time budget in microseconds of the
    tensor-core kernel's inter-role waits (0 = the default, 2 s) and, with
    ``hold_first_tile``, a first key tile that the first CTA of the next
    dense-kind launches never loads, so that a wait runs out and the launch
    reports DSA_ERR_TIMEOUT through the status word.  Process-wide."""
    _check(lib().dsa_debug_set_wait(int(budget_us), 1 if hold_first_tile else 0), "dsa_debug_set_wait")


def _check_out(idx, val, rows, k):
    # the library writes rows * k entries into each: a smaller buffer would overflow
    if idx.dtype != torch.int32 or val.dtype != torch.float32:
        raise TypeError("out must be (int32 idx, float32 val)")
    if tuple(idx.shape) != (rows, k) or tuple(val.shape) != (rows, k):
        raise ValueError(f"out must be two [{rows}, {k}] tensors")


def _outputs(rows, k, device, out):
    if out is not None:
        idx, val = out
        _need_cuda(idx, val)
        _check_out(idx, val, rows, k)
        return idx, val
    return (torch.empty((rows, k), dtype=torch.int32, device=device),
            torch.empty((rows, k), dtype=torch.float32, device=device))


def dsa_index_dense(Q: torch.Tensor, w: torch.Tensor, K: torch.Tensor, k: int, q_pos0: Optional[int] = None,
                    K_scale: Optional[torch.Tensor] = None, out=None, workspace=None, stream=None,
                    check: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Dense prefill indexer: per query row t the top-k keys among 0..q_pos0+t.

    Q [T,H,d] bf16/fp32, w [T,H] fp32, K [N,d] bf16/fp32 or fp8 e4m3 bytes
    (then ``K_scale`` [N] fp32).  Returns (idx [T,k] int32, val [T,k] fp32);
    each row is a set, padded with -1 / -inf.
    """
    _check_shapes(Q, w, K, K_scale)
    _need_cuda(Q, w, K, K_scale)
    T, H, d = Q.shape
    N = K.shape[0]
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    nb = dense_workspace_bytes(T, N, H, d, k, qd, kd)
    ws = _workspace(nb, Q.device, workspace)
    idx, val = _outputs(T, k, Q.device, out)
    _check(lib().dsa_index_dense(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), T, N, H, d, q_pos0, k, qd, kd,
                                 _ptr(idx), _ptr(val), _ptr(ws), ws.numel(), _stream(stream)), "dsa_index_dense")
    if check:
        dsa_check_status(ws, stream)
    return idx, val


def dsa_index_group(Q, w, K, k: int, group: int, bank: int, mode: int = DSA_GROUP_REFINE,
                    q_pos0: Optional[int] = None, K_scale=None, out=None, return_bank: bool = False,
                    return_proxy: bool = False, workspace=None, stream=None, check: bool = False):
    """Group-shared (PIVOT) prefill indexer, Refine or Reuse.

    Returns (idx, val) and, on request, (bank_idx [ng,B], bank_val [ng,B]) in
    the proxy's ranking order and (proxy_q [ng,H,d], proxy_w [ng,H]).
    """
    _check_shapes(Q, w, K, K_scale)
    _need_cuda(Q, w, K, K_scale)
    T, H, d = Q.shape
    N = K.shape[0]
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    ng = (T + group - 1) // group
    nb = group_workspace_bytes(T, N, H, d, k, group, bank, qd, kd)
    ws = _workspace(nb, Q.device, workspace)
    idx, val = _outputs(T, k, Q.device, out)
    bi = bv = pq = pw = None
    if return_bank:
        bi = torch.empty((ng, bank), dtype=torch.int32, device=Q.device)
        bv = torch.empty((ng, bank), dtype=torch.float32, device=Q.device)
    if return_proxy:
        pq = torch.empty((ng, H, d), dtype=Q.dtype, device=Q.device)
        pw = torch.empty((ng, H), dtype=torch.float32, device=Q.device)
    _check(lib().dsa_index_group(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), T, N, H, d, q_pos0, k, group, bank,
                                 int(mode), qd, kd, _ptr(idx), _ptr(val), _ptr(bi), _ptr(bv), _ptr(pq), _ptr(pw),
                                 _ptr(ws), ws.numel(), _stream(stream)), "dsa_index_group")
    if check:
        dsa_check_status(ws, stream)
    res = [idx, val]
    if return_bank:
        res += [bi, bv]
    if return_proxy:
        res += [pq, pw]
    return tuple(res)


def dsa_index_decode(Q, w, K, k: int, k_offsets: torch.Tensor, q_offsets: torch.Tensor,
                     max_keys: Optional[int] = None, total_keys: Optional[int] = None, K_scale=None, out=None,
                     workspace=None, stream=None, check: bool = False):
    """Decode indexer over B key caches; offsets are [B+1] (host or device).

    With device offsets (int64 / int32) and ``max_keys`` / ``total_keys``
    given, the call does no host-side work on the offsets (no copies, no
    synchronisation).  Returns (idx [sum m_b, k], val) with key indices
    local to each sequence.
    """
    _check_shapes(Q, w, K, K_scale)
    _need_cuda(Q, w, K, K_scale)
    total_q, H, d = Q.shape
    B = k_offsets.numel() - 1
    ko, qo, max_keys, total_keys = _decode_offsets(Q, K, k_offsets, q_offsets, max_keys, total_keys)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    nb = decode_workspace_bytes(B, total_q, max_keys, H, d, k, qd, kd)
    ws = _workspace(nb, Q.device, workspace)
    idx, val = _outputs(total_q, k, Q.device, out)
    _check(lib().dsa_index_decode(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), _ptr(ko), _ptr(qo), B, total_q,
                                  int(total_keys), int(max_keys), H, d, k, qd, kd, _ptr(idx), _ptr(val), _ptr(ws),
                                  ws.numel(), _stream(stream)), "dsa_index_decode")
    if check:
        dsa_check_status(ws, stream)
    return idx, val


def decode_group_workspace_bytes(B, total_q, max_keys, H, d, k, bank, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_decode_group_workspace_size(B, total_q, max_keys, H, d, k, bank, q_dtype, k_dtype,
                                                       ctypes.byref(n)), "dsa_index_decode_group_workspace_size")
    return int(n.value)


def _decode_offsets(Q, K, k_offsets, q_offsets, max_keys, total_keys):
    """Offsets on the host (or copied there because max_keys / total_keys are
    missing) are checked here in full: k_offsets[0] = q_offsets[0] = 0,
    q_offsets[B] = Q's rows, k_offsets[B] = total_keys <= K's rows, and every
    sequence with 1 <= N_b <= max_keys keys and 1 <= m_b <= min(4, N_b)
    queries.  Device offsets with both sizes given are not read back (no
    synchronisation); the library checks them on the device and reports an
    invalid argument through the status word."""
    if k_offsets.numel() != q_offsets.numel() or k_offsets.numel() < 1:
        raise ValueError("k_offsets and q_offsets must both be [B+1]")
    if total_keys is not None and int(total_keys) > K.shape[0]:
        raise ValueError(f"total_keys {int(total_keys)} exceeds the {K.shape[0]} rows of K")
    on_host = not (k_offsets.is_cuda and q_offsets.is_cuda)
    if on_host or max_keys is None or total_keys is None:
        ko_h = k_offsets.to("cpu", torch.int64)
        qo_h = q_offsets.to("cpu", torch.int64)
        nb, mb = ko_h[1:] - ko_h[:-1], qo_h[1:] - qo_h[:-1]
        if max_keys is None:
            max_keys = int(nb.max()) if nb.numel() else 0
        if total_keys is None:
            total_keys = int(ko_h[-1])
        bad = None
        if int(ko_h[0]) != 0 or int(qo_h[0]) != 0:
            bad = "offsets must start at 0"
        elif int(qo_h[-1]) != Q.shape[0]:
            bad = f"q_offsets[B] = {int(qo_h[-1])} is not the {Q.shape[0]} query rows"
        elif int(ko_h[-1]) != int(total_keys) or int(total_keys) > K.shape[0]:
            bad = f"k_offsets[B] = {int(ko_h[-1])} must equal total_keys ({int(total_keys)}) <= K's {K.shape[0]} rows"
        elif nb.numel() and (bool((nb < 1).any()) or int(nb.max()) > int(max_keys)):
            bad = f"every sequence needs 1 .. max_keys ({int(max_keys)}) keys"
        elif mb.numel() and (bool((mb < 1).any()) or bool((mb > 4).any()) or bool((mb > nb).any())):
            bad = "every sequence needs 1 <= m_b <= min(4, N_b) new queries"
        if bad:
            raise ValueError(bad)
    ko = k_offsets if (k_offsets.is_cuda and k_offsets.dtype == torch.int64) else \
        k_offsets.to(Q.device, torch.int64).contiguous()
    qo = q_offsets if (q_offsets.is_cuda and q_offsets.dtype == torch.int32) else \
        q_offsets.to(Q.device, torch.int32).contiguous()
    return ko, qo, int(max_keys), int(total_keys)


def dsa_index_decode_group(Q, w, K, k: int, k_offsets: torch.Tensor, q_offsets: torch.Tensor, bank: int,
                           mode: int = DSA_GROUP_REFINE, max_keys: Optional[int] = None,
                           total_keys: Optional[int] = None, K_scale=None, out=None, return_bank: bool = False,
                           return_proxy: bool = False, workspace=None, stream=None, check: bool = False):
    """PIVOT in decode: each sequence's new queries form one group.

    Returns (idx [sum m_b, k], val) with indices local to each sequence and,
    on request, (bank_idx [B, bank], bank_val) in the proxy's ranking order
    and (proxy_q [B, H, d], proxy_w [B, H]).
    """
    _check_shapes(Q, w, K, K_scale)
    _need_cuda(Q, w, K, K_scale)
    total_q, H, d = Q.shape
    B = k_offsets.numel() - 1
    ko, qo, max_keys, total_keys = _decode_offsets(Q, K, k_offsets, q_offsets, max_keys, total_keys)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    nb = decode_group_workspace_bytes(B, total_q, max_keys, H, d, k, bank, qd, kd)
    ws = _workspace(nb, Q.device, workspace)
    idx, val = _outputs(total_q, k, Q.device, out)
    bi = bv = pq = pw = None
    if return_bank:
        bi = torch.empty((B, bank), dtype=torch.int32, device=Q.device)
        bv = torch.empty((B, bank), dtype=torch.float32, device=Q.device)
    if return_proxy:
        pq = torch.empty((B, H, d), dtype=Q.dtype, device=Q.device)
        pw = torch.empty((B, H), dtype=torch.float32, device=Q.device)
    _check(lib().dsa_index_decode_group(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), _ptr(ko), _ptr(qo), B, total_q,
                                        total_keys, max_keys, H, d, k, bank, int(mode), qd, kd, _ptr(idx),
                                        _ptr(val), _ptr(bi), _ptr(bv), _ptr(pq), _ptr(pw), _ptr(ws), ws.numel(),
                                        _stream(stream)), "dsa_index_decode_group")
    if check:
        dsa_check_status(ws, stream)
    res = [idx, val]
    if return_bank:
        res += [bi, bv]
    if return_proxy:
        res += [pq, pw]
    return tuple(res)


def block_routed_workspace_bytes(T, N, H, d, k, n_blocks, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_block_routed_workspace_size(T, N, H, d, k, n_blocks, q_dtype, k_dtype, ctypes.byref(n)),
           "dsa_index_block_routed_workspace_size")
    return int(n.value)


def dsa_index_block_routed(Q, w, K, k: int, n_blocks: int, q_pos0: Optional[int] = None, K_scale=None, out=None,
                           return_blocks: bool = False, return_reps: bool = False, workspace=None, stream=None,
                           check: bool = False):
    """Two-stage selection over 128-key blocks (block routing), then the native score.

    Returns (idx, val) and, on request, the routed blocks [T, n_blocks] and
    the block representatives [ceil(N/128), d] (bf16).
    """
    _check_shapes(Q, w, K, K_scale)
    _need_cuda(Q, w, K, K_scale)
    T, H, d = Q.shape
    N = K.shape[0]
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    nb = block_routed_workspace_bytes(T, N, H, d, k, n_blocks, qd, kd)
    ws = _workspace(nb, Q.device, workspace)
    idx, val = _outputs(T, k, Q.device, out)
    bi = torch.empty((T, n_blocks), dtype=torch.int32, device=Q.device) if return_blocks else None
    rp = torch.empty(((N + 127) // 128, d), dtype=torch.bfloat16, device=Q.device) if return_reps else None
    _check(lib().dsa_index_block_routed(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), T, N, H, d, q_pos0, k, n_blocks,
                                        qd, kd, _ptr(idx), _ptr(val), _ptr(bi), _ptr(rp), _ptr(ws), ws.numel(),
                                        _stream(stream)), "dsa_index_block_routed")
    if check:
        dsa_check_status(ws, stream)
    res = [idx, val]
    if return_blocks:
        res.append(bi)
    if return_reps:
        res.append(rp)
    return tuple(res)


class IvfIndex:
    """A plain k-means inverted-file index of the keys (device buffer owned by torch).

    Parts (views into ``buffer``): off [C+1], perm [N] (clustered row -> key),
    assign [N], keys [N, d] bf16 (clustered), centroids_bf16 [C, d],
    centroids [C, d] fp32.
    """

    def __init__(self, buffer: torch.Tensor, N: int, d: int, C: int):
        self.buffer, self.N, self.d, self.C = buffer, N, d, C
        o = 0
        parts = {}
        for name, nbytes in (("off", (C + 1) * 4), ("perm", N * 4), ("assign", N * 4), ("keys", N * d * 2),
                             ("centroids_bf16", C * d * 2), ("centroids", C * d * 4)):
            parts[name] = (o, nbytes)
            o += (nbytes + 255) // 256 * 256
        self._parts = parts
        self.max_cluster_tiles = None

    def part(self, name):
        o, n = self._parts[name]
        raw = self.buffer[o:o + n]
        if name in ("off", "perm", "assign"):
            return raw.view(torch.int32)
        if name in ("keys", "centroids_bf16"):
            return raw.view(torch.bfloat16).view(-1, self.d)
        return raw.view(torch.float32).view(-1, self.d)

    def probe_tile_bound(self, n_probe: int) -> int:
        """Tiles of the n_probe largest clusters (a bound for any query's probe)."""
        if self.max_cluster_tiles is None:
            off = self.part("off").cpu().numpy().astype(np.int64)
            self.max_cluster_tiles = np.sort(-(-(off[1:] - off[:-1]) // 128))[::-1]
        return max(1, int(self.max_cluster_tiles[:n_probe].sum()))


def dsa_ivf_build(K, C: int, iters: int = 10, K_scale=None, stream=None, check: bool = False) -> IvfIndex:
    """Plain k-means index of the keys (Lloyd, `iters` iterations) for inverted-file routing."""
    _check_shapes(None, None, K, K_scale)
    _need_cuda(K, K_scale)
    N, d = K.shape
    kd = _dtype_code(K, allow_fp8=True)
    nb = ctypes.c_size_t(0)
    _check(lib().dsa_ivf_index_size(N, d, C, ctypes.byref(nb)), "dsa_ivf_index_size")
    buf = torch.zeros(int(nb.value), dtype=torch.uint8, device=K.device)
    wb = ctypes.c_size_t(0)
    _check(lib().dsa_ivf_build_workspace_size(N, 64, d, C, DSA_DTYPE_BF16, kd, ctypes.byref(wb)),
           "dsa_ivf_build_workspace_size")
    ws = torch.zeros(max(int(wb.value), 256), dtype=torch.uint8, device=K.device)
    _check(lib().dsa_ivf_build(_ptr(K), _ptr(K_scale), N, 64, d, C, iters, DSA_DTYPE_BF16, kd, _ptr(buf), buf.numel(),
                               _ptr(ws), ws.numel(), _stream(stream)), "dsa_ivf_build")
    if check:
        dsa_check_status(ws, stream)
    return IvfIndex(buf, N, d, C)


def ivf_routed_workspace_bytes(T, N, H, d, k, C, n_probe, max_tiles, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_ivf_routed_workspace_size(T, N, H, d, k, C, n_probe, max_tiles, q_dtype, k_dtype,
                                                     ctypes.byref(n)), "dsa_index_ivf_routed_workspace_size")
    return int(n.value)


def dsa_index_ivf_routed(Q, w, index: IvfIndex, k: int, n_probe: int, q_pos0: Optional[int] = None, K_scale=None,
                         max_tiles: Optional[int] = None, out=None, return_clusters: bool = False, workspace=None,
                         stream=None, check: bool = False):
    """Inverted-file routing over `index`, then the native score on the probed clusters' keys."""
    _check_shapes(Q, w, None, K_scale, index.N)
    _need_cuda(Q, w, K_scale)
    T, H, d = Q.shape
    N, C = index.N, index.C
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    qd = _dtype_code(Q)
    kd = DSA_DTYPE_FP8_E4M3 if K_scale is not None else DSA_DTYPE_BF16
    mt = index.probe_tile_bound(n_probe) if max_tiles is None else int(max_tiles)
    ws = _workspace(ivf_routed_workspace_bytes(T, N, H, d, k, C, n_probe, mt, qd, kd), Q.device, workspace)
    idx, val = _outputs(T, k, Q.device, out)
    ci = torch.empty((T, n_probe), dtype=torch.int32, device=Q.device) if return_clusters else None
    _check(lib().dsa_index_ivf_routed(_ptr(Q), _ptr(w), _ptr(index.buffer), _ptr(K_scale), T, N, H, d, q_pos0, k, C,
                                      n_probe, mt, qd, kd, _ptr(idx), _ptr(val), _ptr(ci), _ptr(ws), ws.numel(),
                                      _stream(stream)), "dsa_index_ivf_routed")
    if check:
        dsa_check_status(ws, stream)
    return (idx, val, ci) if return_clusters else (idx, val)


def dsa_debug_scores(Q, w, K, q_pos0: Optional[int] = None, K_scale=None, workspace=None, stream=None,
                     check: bool = False) -> torch.Tensor:
    """Test aid: the full [T, N] score matrix of the dense kernels (-inf beyond each prefix)."""
    _check_shapes(Q, w, K, K_scale)
    _need_cuda(Q, w, K, K_scale)
    T, H, d = Q.shape
    N = K.shape[0]
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    nb = dense_workspace_bytes(T, N, H, d, 1, qd, kd) + 8 * T + 1024
    ws = _workspace(nb, Q.device, workspace)
    S = torch.empty((T, N), dtype=torch.float32, device=Q.device)
    _check(lib().dsa_debug_scores(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), T, N, H, d, q_pos0, qd, kd, _ptr(S),
                                  _ptr(ws), ws.numel(), _stream(stream)), "dsa_debug_scores")
    if check:
        dsa_check_status(ws, stream)
    return S


def dsa_index_dense_static(Q: torch.Tensor, w: torch.Tensor, K: torch.Tensor, k: int, q_pos0: Optional[int] = None,
                           out=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Dense indexer that allocates no device memory (bf16 Q/K, H = 64, d = 128).

    For callers that cannot provide a workspace: the library's fixed scratch
    array is used instead.  Synchronous; calls on one device must not
    overlap.  ``out`` = (idx, val) preallocated by the caller, else
    allocated here (by torch, outside the library).
    """
    _check_shapes(Q, w, K)
    _need_cuda(Q, w, K)
    T, H, d = Q.shape
    N = K.shape[0]
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    if Q.dtype != torch.bfloat16 or K.dtype != torch.bfloat16:
        raise TypeError("dsa_index_dense_static takes bf16 Q and K")
    idx, val = _outputs(T, k, Q.device, out)
    _check(lib().dsa_index_dense_static(_ptr(Q), _ptr(w), _ptr(K), T, N, H, d, q_pos0, k, _ptr(idx), _ptr(val),
                                        _stream(stream)), "dsa_index_dense_static")
    return idx, val


def dsa_kernel_timer_start(max_launches: int) -> None:
    """Arm the library's scoring-kernel timer for up to ``max_launches`` launches."""
    _check(lib().dsa_kernel_timer_start(int(max_launches)), "dsa_kernel_timer_start")


def dsa_kernel_timer_stop() -> Tuple[float, int]:
    """Disarm the timer; (summed kernel milliseconds, timed launches)."""
    ms, n = ctypes.c_float(0.0), _c_int(0)
    _check(lib().dsa_kernel_timer_stop(ctypes.byref(ms), ctypes.byref(n)), "dsa_kernel_timer_stop")
    return float(ms.value), int(n.value)


# ---------------------------------------------------------------------------
# host-buffer entry points: inputs and outputs in host memory (page-locked for
# overlap), staged through a device buffer; synchronous
# ---------------------------------------------------------------------------
def _need_host(*ts):
    for t in ts:
        if t is None:
            continue
        if t.is_cuda:
            raise ValueError("host-buffer call: tensors must be in host memory")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _host_outputs(rows: int, k: int, out):
    if out is not None:
        _need_host(*out)
        _check_out(out[0], out[1], rows, k)
        return out
    return (torch.empty((rows, k), dtype=torch.int32).pin_memory(),
            torch.empty((rows, k), dtype=torch.float32).pin_memory())


def _staging(nbytes: int, device, staging):
    if staging is not None:
        if not staging.is_cuda or staging.numel() * staging.element_size() < nbytes:
            raise ValueError(f"staging must be a device buffer of at least {nbytes} bytes")
        return staging
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)


def dense_host_staging_bytes(T, N, H, d, k, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_dense_host_staging_size(T, N, H, d, k, q_dtype, k_dtype, ctypes.byref(n)),
           "dsa_index_dense_host_staging_size")
    return int(n.value)


def group_host_staging_bytes(T, N, H, d, k, group, bank, q_dtype, k_dtype, chunk_rows=0) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_group_host_staging_size(T, N, H, d, k, group, bank, q_dtype, k_dtype, chunk_rows,
                                                   ctypes.byref(n)), "dsa_index_group_host_staging_size")
    return int(n.value)


def decode_host_staging_bytes(B, total_q, total_keys, max_keys, H, d, k, q_dtype, k_dtype) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dsa_index_decode_host_staging_size(B, total_q, total_keys, max_keys, H, d, k, q_dtype, k_dtype,
                                                    ctypes.byref(n)), "dsa_index_decode_host_staging_size")
    return int(n.value)


def dsa_index_dense_host(Q, w, K, k: int, q_pos0: Optional[int] = None, K_scale=None, out=None,
                         chunk_rows: int = 0, staging=None, device=None, stream=None):
    """Dense indexer on host tensors; returns host (idx [T,k], val [T,k]).

    The inputs are copied in and the outputs out in row chunks that overlap
    the indexer; ``staging`` is an optional device uint8 buffer of at least
    ``dense_host_staging_bytes`` bytes.  Returns once the outputs are filled.
    """
    _check_shapes(Q, w, K, K_scale)
    _need_host(Q, w, K, K_scale)
    T, H, d = Q.shape
    N = K.shape[0]
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    st = _staging(dense_host_staging_bytes(T, N, H, d, k, qd, kd), device, staging)
    idx, val = _host_outputs(T, k, out)
    with torch.cuda.device(st.device):
        _check(lib().dsa_index_dense_host(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), T, N, H, d, q_pos0, k, qd, kd,
                                          int(chunk_rows), _ptr(idx), _ptr(val), _ptr(st), st.numel(),
                                          _stream(stream)), "dsa_index_dense_host")
    return idx, val


def dsa_index_group_host(Q, w, K, k: int, group: int, bank: int, mode: int = DSA_GROUP_REFINE,
                         q_pos0: Optional[int] = None, K_scale=None, out=None, chunk_rows: int = 0, staging=None,
                         device=None, stream=None):
    """Group-shared (PIVOT) indexer on host tensors; returns host (idx, val).

    Chunks hold whole groups, so the results equal one call over all rows.
    """
    _check_shapes(Q, w, K, K_scale)
    _need_host(Q, w, K, K_scale)
    T, H, d = Q.shape
    N = K.shape[0]
    q_pos0 = N - T if q_pos0 is None else int(q_pos0)
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    st = _staging(group_host_staging_bytes(T, N, H, d, k, group, bank, qd, kd, int(chunk_rows)), device, staging)
    idx, val = _host_outputs(T, k, out)
    with torch.cuda.device(st.device):
        _check(lib().dsa_index_group_host(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), T, N, H, d, q_pos0, k, group,
                                          bank, mode, qd, kd, int(chunk_rows), _ptr(idx), _ptr(val), _ptr(st),
                                          st.numel(), _stream(stream)), "dsa_index_group_host")
    return idx, val


def dsa_index_decode_host(Q, w, K, k: int, k_offsets: torch.Tensor, q_offsets: torch.Tensor,
                          max_keys: Optional[int] = None, K_scale=None, out=None, staging=None, device=None,
                          stream=None):
    """Decode indexer on host tensors and host offsets ([B+1] int64 / int32);
    returns host (idx [sum m_b, k], val) with key indices local to each
    sequence."""
    _check_shapes(Q, w, K, K_scale)
    _need_host(Q, w, K, K_scale, k_offsets, q_offsets)
    if k_offsets.numel() != q_offsets.numel() or k_offsets.numel() < 1:
        raise ValueError("k_offsets and q_offsets must both be [B+1]")
    total_q, H, d = Q.shape
    B = k_offsets.numel() - 1
    ko = k_offsets.to(torch.int64).contiguous()
    qo = q_offsets.to(torch.int32).contiguous()
    total_keys = int(ko[-1])
    if max_keys is None:
        max_keys = int((ko[1:] - ko[:-1]).max()) if ko.numel() > 1 else 0
    _decode_offsets(Q, K, ko, qo, max_keys, total_keys)  # host offsets: checked in full
    qd, kd = _dtype_code(Q), _dtype_code(K, allow_fp8=True)
    st = _staging(decode_host_staging_bytes(B, total_q, total_keys, max_keys, H, d, k, qd, kd), device, staging)
    idx, val = _host_outputs(total_q, k, out)
    with torch.cuda.device(st.device):
        _check(lib().dsa_index_decode_host(_ptr(Q), _ptr(w), _ptr(K), _ptr(K_scale), _ptr(ko), _ptr(qo), B,
                                           total_q, total_keys, int(max_keys), H, d, k, qd, kd, _ptr(idx), _ptr(val),
                                           _ptr(st), st.numel(), _stream(stream)), "dsa_index_decode_host")
    return idx, val
