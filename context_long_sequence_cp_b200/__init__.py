"""Context-parallel attention on one B200: Python binding of ``libcp_attn.so``.

This module only marshals arguments: every step of the computation runs in the
CUDA library built from ``csrc/`` (see ``include/cp_attn.h`` for the C ABI). It
uses PyTorch for device memory and streams. There is no CPU fallback: importing
raises when the library is missing, and every call raises on a non-zero status.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcp_attn.so")

CONTIGUOUS, ZIGZAG, ULYSSES = 0, 1, 2
LAYOUTS = {"contiguous": CONTIGUOUS, "zigzag": ZIGZAG, "ulysses": ULYSSES}

STATUS = {0: "CP_OK", -1: "CP_ERR_INVALID_ARG", -2: "CP_ERR_UNSUPPORTED", -3: "CP_ERR_ALIGNMENT",
          -4: "CP_ERR_CUDA", -5: "CP_ERR_TIMEOUT", -6: "CP_ERR_WORKSPACE"}

# Every function the header declares, with its ctypes signature.
_P, _I, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "cp_attn_plan": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I, _F]),
    "cp_attn_plan_destroy": (_I, [_P]),
    "cp_attn_plan_tile_counts": (_I64, [_P, _P]),
    "cp_attn_plan_num_items": (_I64, [_P]),
    "cp_attn_plan_cta_loads": (_I64, [_P, _P]),
    "cp_attn_bwd": (_I, [_P] * 12),
    "cp_sp_rs_dropout_add_ln": (_I, [_P, _I, _I64, _I, _P, ctypes.c_float, _P, _P, _P, ctypes.c_float, _P, _P, _P]),
    "cp_attn_bwd_workspace_bytes": (ctypes.c_size_t, [_P]),
    "cp_attn_plan_bwd_pairs": (_I64, [_P, _P, _P]),
    "cp_attn_workspace_bytes": (_SZ, [_P, _I]),
    "cp_attn_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "cp_attn_fwd_partials": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "cp_merge_partials": (_I, [_I, _I64, _I, _P, _P, _P, _P, _P]),
    "cp_layout_permute": (_I, [_P, _I, _P, _P, _I, _P]),
    "cp_rope_permute": (_I, [_P, _P, _P, ctypes.c_double, _I64, _P]),
    "cp_layout_index_map_len": (_I64, [_P]),
    "cp_layout_index_map": (_I, [_P, _P, _P]),
    "cp_attn_check": (_I, [_P, _P]),
    "cp_status_string": (ctypes.c_char_p, [_I]),
    "cp_debug_wait_timeout_probe": (_I, [_P, _I, _P]),
    "cp_attn_fwd_ulysses_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P]),
    "cp_attn_fwd_ring_step": (_I, [_P, _I, _I, _P, _P, _P, _P, _P, _P]),
    "cp_attn_ring_prepare": (_I, [_P, _I]),
    "cp_attn_ring_num_parts": (_I, [_P]),
    "cp_attn_fwd_ring": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "cp_attn_fwd_ring_external": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P]),
    "cp_attn_ring_schedule": (_I64, [_P, _I, _I, _P, _P]),
    "cp_ring_buffer_alloc": (_I, [_SZ, ctypes.POINTER(_P)]),
    "cp_ring_buffer_free": (_I, [_P]),
    "cp_ipc_handle_bytes": (_I, []),
    "cp_ipc_get_handle": (_I, [_P, _P]),
    "cp_ipc_open_handle": (_I, [_P, ctypes.POINTER(_P)]),
    "cp_ipc_close_handle": (_I, [_P]),
    "cp_copy_async": (_I, [_P, _P, _SZ, _P]),
}

# Size of the library's fixed device scratch used by the no-alloc Ulysses
# forward (CP_NOALLOC_SCRATCH_BYTES in include/cp_attn.h).
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class CpAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({lib().cp_status_string(status).decode()})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m context_long_sequence_cp_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise CpAttnError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


class Plan:
    """A context-parallel attention plan (wraps ``cp_attn_plan``)."""

    def __init__(self, B: int, H: int, S: int, D: int, N: int, causal: bool, layout: str = "zigzag",
                 softmax_scale: float = 0.0):
        self.B, self.H, self.S, self.D, self.N = B, H, S, D, N
        self.causal, self.layout = bool(causal), layout
        self.scale = softmax_scale if softmax_scale > 0 else 1.0 / math.sqrt(D)
        h = ctypes.c_void_p()
        _check("cp_attn_plan", lib().cp_attn_plan(ctypes.byref(h), B, H, S, D, N, int(bool(causal)),
                                                   LAYOUTS[layout], float(softmax_scale)))
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().cp_attn_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def tile_counts(self):
        arr = (ctypes.c_int64 * self.N)()
        tot = lib().cp_attn_plan_tile_counts(self._h, ctypes.cast(arr, ctypes.c_void_p))
        if tot < 0:
            raise CpAttnError("cp_attn_plan_tile_counts", int(tot))
        return list(arr), int(tot)

    def num_items(self) -> int:
        return int(lib().cp_attn_plan_num_items(self._h))

    def bwd_pairs(self):
        """(key-tile walk pairs, query-tile walk pairs) of the backward, per (batch, head)."""
        kv, qq = ctypes.c_int64(0), ctypes.c_int64(0)
        rc = int(lib().cp_attn_plan_bwd_pairs(self._h, ctypes.byref(kv), ctypes.byref(qq)))
        if rc < 0:
            raise CpAttnError("cp_attn_plan_bwd_pairs", rc)
        return int(kv.value), int(qq.value)

    def bwd_workspace_bytes(self) -> int:
        return int(lib().cp_attn_bwd_workspace_bytes(self._h))

    def cta_loads(self):
        """Modelled load of each CTA of the kernel's static schedule."""
        n = int(lib().cp_attn_plan_cta_loads(self._h, None))
        if n < 0:
            raise CpAttnError("cp_attn_plan_cta_loads", n)
        arr = (ctypes.c_int64 * max(n, 1))()
        lib().cp_attn_plan_cta_loads(self._h, ctypes.cast(arr, ctypes.c_void_p))
        return list(arr)[:n]

    def ring_prepare(self, rank: int):
        """Build (and upload) the per-step schedules of one rank's ring steps."""
        _check("cp_attn_ring_prepare", lib().cp_attn_ring_prepare(self._h, int(rank)))

    def ring_parts(self) -> int:
        """Number of partials of the one-launch ring forward."""
        n = int(lib().cp_attn_ring_num_parts(self._h))
        if n < 0:
            raise CpAttnError("cp_attn_ring_num_parts", n)
        return n

    def ring_schedule(self, rank: int, step: int):
        """Schedule of one rank's ring step: (items as rows of (row block, head,
        query-tile pair, key tiles, CTA) in run order, per-CTA modelled loads);
        step -1: the units of the one-launch ring forward (pair | first step << 16 |
    end step << 24)."""
        n = int(lib().cp_attn_ring_schedule(self._h, int(rank), int(step), None, None))
        if n < 0:
            raise CpAttnError("cp_attn_ring_schedule", n)
        items = (ctypes.c_int32 * (5 * n))()
        loads = (ctypes.c_int64 * max(n, 1))()
        lib().cp_attn_ring_schedule(self._h, int(rank), int(step), ctypes.cast(items, ctypes.c_void_p),
                                    ctypes.cast(loads, ctypes.c_void_p))
        rows = [tuple(items[5 * i:5 * i + 5]) for i in range(n)]
        n_cta = max(r[4] for r in rows) + 1 if rows else 0
        return rows, list(loads)[:n_cta]

    def workspace_bytes(self, with_partials: bool = False) -> int:
        return int(lib().cp_attn_workspace_bytes(self._h, int(with_partials)))

    def index_map_len(self) -> int:
        return int(lib().cp_layout_index_map_len(self._h))

    @property
    def rows(self) -> int:
        return self.B * self.S * self.H


def attn_fwd(plan: Plan, q, k, v, o=None, lse=None, workspace=None, stream=None):
    """Fused forward (``cp_attn_fwd``): returns (o, lse)."""
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(plan.B, plan.H, plan.S, dtype=torch.float32, device=q.device)
    nws = plan.workspace_bytes(False)
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=q.device)
    _check("cp_attn_fwd", lib().cp_attn_fwd(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                            _ptr(workspace), _stream(stream)))
    return o, lse


def attn_fwd_partials(plan: Plan, q, k, v, o_parts=None, lse_parts=None, stream=None):
    """Per-ring-step partials (``cp_attn_fwd_partials``): ([N, rows, D] fp32, [N, rows] fp32)."""
    if o_parts is None:
        o_parts = torch.empty(plan.N, plan.rows, plan.D, dtype=torch.float32, device=q.device)
    if lse_parts is None:
        lse_parts = torch.empty(plan.N, plan.rows, dtype=torch.float32, device=q.device)
    _check("cp_attn_fwd_partials", lib().cp_attn_fwd_partials(plan.handle, _ptr(q), _ptr(k), _ptr(v),
                                                              _ptr(o_parts), _ptr(lse_parts), None,
                                                              _stream(stream)))
    return o_parts, lse_parts


def attn_fwd_ring_step(plan: Plan, rank: int, step: int, q, k, v, o_part=None, lse_part=None, stream=None):
    """``cp_attn_fwd_ring_step``: rank ``rank``'s partial against the key/value block
    of rank (rank + step) mod N, all buffers rank-local [B, S/N, H, D].
    Returns (o_part fp32 [rows, D], lse_part fp32 [rows]), rows = B*(S/N)*H."""
    rows = plan.B * (plan.S // plan.N) * plan.H
    if o_part is None:
        o_part = torch.empty(rows, plan.D, dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty(rows, dtype=torch.float32, device=q.device)
    _check("cp_attn_fwd_ring_step",
           lib().cp_attn_fwd_ring_step(plan.handle, int(rank), int(step), _ptr(q), _ptr(k), _ptr(v), _ptr(o_part),
                                       _ptr(lse_part), _stream(stream)))
    return o_part, lse_part


def attn_fwd_ring(plan: Plan, rank: int, q, k_all, v_all, pull_k=None, pull_v=None, arrived=None,
                  o_parts=None, lse_parts=None, stream=None):
    """``cp_attn_fwd_ring``: all N step partials of rank ``rank`` in one launch.

    k_all, v_all: [N, B, S/N, H, D] tensors or device addresses (slot j = rank
    j's block; slot ``rank`` filled). pull_k, pull_v: N device addresses of the
    ranks' own blocks to fetch from (None: every slot already filled). arrived:
    int32 [N] device tensor (needed when pulling). Returns (o_parts fp32
    [P, rows, D], lse_parts fp32 [P, rows]), P = plan.ring_parts(),
    rows = B*(S/N)*H."""
    rows = plan.B * (plan.S // plan.N) * plan.H
    P = plan.ring_parts()
    if o_parts is None:
        o_parts = torch.empty(P, rows, plan.D, dtype=torch.float32, device=q.device)
    if lse_parts is None:
        lse_parts = torch.empty(P, rows, dtype=torch.float32, device=q.device)
    pk = None if pull_k is None else (ctypes.c_void_p * len(pull_k))(*[int(x) for x in pull_k])
    pv = None if pull_v is None else (ctypes.c_void_p * len(pull_v))(*[int(x) for x in pull_v])
    as_ptr = lambda a: None if a is None else ctypes.cast(a, ctypes.c_void_p)
    _check("cp_attn_fwd_ring",
           lib().cp_attn_fwd_ring(plan.handle, int(rank), _ptr(q), _vp_of(k_all), _vp_of(v_all), as_ptr(pk),
                                  as_ptr(pv), None if arrived is None else _vp_of(arrived), _ptr(o_parts),
                                  _ptr(lse_parts), _stream(stream)))
    return o_parts, lse_parts


def attn_fwd_ring_external(plan: Plan, rank: int, q, k_all, v_all, arrived, o_parts=None, lse_parts=None,
                           stream=None):
    """``cp_attn_fwd_ring_external``: as ``attn_fwd_ring`` without pull sources,
    each unit waiting (bounded) until ``arrived[j] >= 1`` before it reads slot j;
    the caller's own transfer fills the slots and raises the counts."""
    rows = plan.B * (plan.S // plan.N) * plan.H
    P = plan.ring_parts()
    if o_parts is None:
        o_parts = torch.empty(P, rows, plan.D, dtype=torch.float32, device=q.device)
    if lse_parts is None:
        lse_parts = torch.empty(P, rows, dtype=torch.float32, device=q.device)
    _check("cp_attn_fwd_ring_external",
           lib().cp_attn_fwd_ring_external(plan.handle, int(rank), _ptr(q), _vp_of(k_all), _vp_of(v_all),
                                           _vp_of(arrived), _ptr(o_parts), _ptr(lse_parts), _stream(stream)))
    return o_parts, lse_parts


def _vp_of(x):
    return ctypes.c_void_p(int(x) if isinstance(x, int) else x.data_ptr())


def copy_async(dst_ptr: int, src_ptr: int, nbytes: int, stream=None):
    """``cp_copy_async``: one device-to-device copy (a peer's memory included)."""
    _check("cp_copy_async", lib().cp_copy_async(ctypes.c_void_p(int(dst_ptr)), ctypes.c_void_p(int(src_ptr)),
                                                 int(nbytes), _stream(stream)))


class DeviceBuffer:
    """Device memory from ``cp_ring_buffer_alloc`` (shareable with other processes
    through CUDA IPC), viewable as a torch tensor without a copy."""

    def __init__(self, nbytes: int):
        p = ctypes.c_void_p()
        _check("cp_ring_buffer_alloc", lib().cp_ring_buffer_alloc(int(nbytes), ctypes.byref(p)))
        self.ptr, self.nbytes = int(p.value), int(nbytes)

    def ipc_handle(self) -> bytes:
        buf = ctypes.create_string_buffer(int(lib().cp_ipc_handle_bytes()))
        _check("cp_ipc_get_handle", lib().cp_ipc_get_handle(ctypes.c_void_p(self.ptr), buf))
        return buf.raw

    def view(self, shape, dtype=torch.bfloat16, offset_bytes: int = 0, device=None):
        return _device_view(self.ptr + offset_bytes, shape, dtype, device)

    def close(self):
        if getattr(self, "ptr", 0):
            lib().cp_ring_buffer_free(ctypes.c_void_p(self.ptr))
            self.ptr = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class PeerBuffer:
    """Another process's ``DeviceBuffer`` mapped into this one (``cp_ipc_open_handle``)."""

    def __init__(self, handle: bytes, nbytes: int):
        p = ctypes.c_void_p()
        _check("cp_ipc_open_handle", lib().cp_ipc_open_handle(ctypes.c_char_p(handle), ctypes.byref(p)))
        self.ptr, self.nbytes = int(p.value), int(nbytes)

    def close(self):
        if getattr(self, "ptr", 0):
            lib().cp_ipc_close_handle(ctypes.c_void_p(self.ptr))
            self.ptr = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


_TYPESTR = {torch.bfloat16: "<V2", torch.float32: "<f4", torch.int32: "<i4", torch.uint8: "|u1"}


class _CudaArray:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (int(ptr), False),
                                         "version": 3, "strides": None}


def _device_view(ptr: int, shape, dtype, device=None):
    """A torch tensor over device memory at ``ptr`` (no copy; the memory's owner
    must outlive it)."""
    if dtype == torch.bfloat16:
        t = torch.as_tensor(_CudaArray(ptr, shape, "<i2"), device=device)
        return t.view(torch.bfloat16)
    return torch.as_tensor(_CudaArray(ptr, shape, _TYPESTR[dtype]), device=device)


def merge_partials(o_parts, lse_parts, o_out=None, lse_out=None, stream=None):
    """Merge [P, rows, D] fp32 partials (``cp_merge_partials``): (bf16 [rows, D], fp32 [rows])."""
    P, rows, D = o_parts.shape
    if o_out is None:
        o_out = torch.empty(rows, D, dtype=torch.bfloat16, device=o_parts.device)
    if lse_out is None:
        lse_out = torch.empty(rows, dtype=torch.float32, device=o_parts.device)
    _check("cp_merge_partials", lib().cp_merge_partials(P, rows, D, _ptr(o_parts), _ptr(lse_parts),
                                                        _ptr(o_out), _ptr(lse_out), _stream(stream)))
    return o_out, lse_out


def layout_permute(plan: Plan, x, direction: int, out=None, stream=None):
    """Index-mapped layout copy (``cp_layout_permute``); bit-exact."""
    if out is None:
        out = torch.empty_like(x)
    _check("cp_layout_permute", lib().cp_layout_permute(plan.handle, int(direction), _ptr(x), _ptr(out),
                                                        x.element_size(), _stream(stream)))
    return out


def rope_permute(plan: Plan, x, out=None, base: float = 10000.0, pos_offset: int = 0, stream=None):
    """``cp_rope_permute``: rotary embedding at global positions fused into the
    forward layout map (natural or Ulysses shards -> the attention input layout)."""
    if x.dtype != torch.bfloat16:
        raise CpAttnError("cp_rope_permute", -1)
    if out is None:
        if plan.layout == "ulysses":
            B, H, S, D, N = plan.B, plan.H, plan.S, plan.D, plan.N
            out = torch.empty(N, B, S, H // N, D, dtype=x.dtype, device=x.device)
        else:
            out = torch.empty_like(x)
    _check("cp_rope_permute", lib().cp_rope_permute(plan.handle, _ptr(x), _ptr(out), float(base), int(pos_offset),
                                                    _stream(stream)))
    return out


def attn_bwd(plan: Plan, q, k, v, o, lse, dout, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """``cp_attn_bwd``: (dq, dk, dv) in the plan's attention input layout."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(max(plan.bwd_workspace_bytes(), 16), dtype=torch.uint8, device=q.device)
    _check("cp_attn_bwd", lib().cp_attn_bwd(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), _stream(stream)))
    return dq, dk, dv


def sp_rs_dropout_add_ln(partials, keep_bits=None, p: float = 0.0, residual=None, gamma=None, beta=None,
                         eps: float = 1e-5, z=None, y=None, want_z=True, want_y=True, stream=None):
    """``cp_sp_rs_dropout_add_ln``: z = dropout(sum of partials) + residual, y = LayerNorm(z).

    partials: bf16 [nparts, rows, H]; keep_bits: int32/uint32 tensor of packed keep bits."""
    nparts, rows, H = partials.shape
    if want_z and z is None:
        z = torch.empty(rows, H, dtype=torch.bfloat16, device=partials.device)
    if want_y and gamma is not None and y is None:
        y = torch.empty(rows, H, dtype=torch.bfloat16, device=partials.device)
    _check("cp_sp_rs_dropout_add_ln",
           lib().cp_sp_rs_dropout_add_ln(_ptr(partials), int(nparts), int(rows), int(H),
                                         _ptr(keep_bits) if keep_bits is not None else None, float(p),
                                         _ptr(residual) if residual is not None else None,
                                         _ptr(gamma) if gamma is not None else None,
                                         _ptr(beta) if beta is not None else None, float(eps),
                                         _ptr(z) if z is not None else None, _ptr(y) if y is not None else None,
                                         _stream(stream)))
    return z, y


def layout_index_map(plan: Plan, device="cuda", stream=None):
    """The layout's int64 index map (``cp_layout_index_map``)."""
    out = torch.empty(plan.index_map_len(), dtype=torch.int64, device=device)
    _check("cp_layout_index_map", lib().cp_layout_index_map(plan.handle, _ptr(out), _stream(stream)))
    return out


def check(plan: Plan, stream=None) -> int:
    """``cp_attn_check``: synchronise and return the recorded status (0 = ok)."""
    return int(lib().cp_attn_check(plan.handle, _stream(stream)))


def debug_wait_timeout_probe(plan: Plan, timeout_us: int, stream=None):
    _check("cp_debug_wait_timeout_probe",
           lib().cp_debug_wait_timeout_probe(plan.handle, int(timeout_us), _stream(stream)))


def attn_fwd_ulysses_noalloc(plan: Plan, q, k, v, o, lse=None, stream=None):
    """Ulysses forward that allocates nothing (``cp_attn_fwd_ulysses_noalloc``).

    For callers that cannot allocate device memory at call time: the head-group
    copies live in the library's fixed 32 MiB device scratch instead of a
    workspace, so ``o`` (and ``lse`` if wanted) must be passed in. Calls that
    may overlap on the GPU share that scratch and must be serialised.
    """
    if plan.layout != "ulysses":
        raise ValueError("attn_fwd_ulysses_noalloc needs a Ulysses plan")
    B, H, S, D, N = plan.B, plan.H, plan.S, plan.D, plan.N
    shape = (N, B, S // N, H, D)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous() or t.device.type != "cuda":
            raise ValueError(f"{name}: expected a contiguous bf16 CUDA tensor of shape {shape}")
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, S) or not lse.is_contiguous()
                            or lse.device != o.device):
        raise ValueError(f"lse: expected a contiguous float32 tensor of shape {(B, H, S)} on {o.device}")
    if any(t.device != o.device for t in (q, k, v)):
        raise ValueError("q, k, v and o must be on one device")
    _check("cp_attn_fwd_ulysses_noalloc",
           lib().cp_attn_fwd_ulysses_noalloc(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                            _stream(stream)))
    return o, lse


def status_string(status: int) -> str:
    return lib().cp_status_string(int(status)).decode()
