"""Python binding of the C ABI in ``include/dspark_verify.h`` (argument marshalling only).

The names follow the dspark-mlx wheel's verify module (page "dspark-mlx
0.1.0__py3-none-any.whl", ``dspark_mlx/__init__.py``: ``AcceptResult``, ``greedy_accept``,
``speculative_sample_accept``). Every step of the verify runs in the CUDA library; this
module only checks tensor layouts, allocates the result tensors and a workspace with
PyTorch, and passes raw device pointers and the current CUDA stream. There is no CPU
fallback: without the built library or a CUDA device every call raises.

Logit inputs follow the wheel's block convention (``dspark_mlx/adapter.py``): either the
full ``[B, K+1, V]`` block, or the pair ``(p1, pv)`` with ``p1 = StepOut.logits`` ``[B, V]``
and ``pv = BlockOut.per_pos_logits`` ``[B, K, V]``, passed without concatenation.
"""

from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional, Tuple, Union

import torch

from . import build_lib

DSPARK_OK = 0
STATIC_SCRATCH_BYTES = 4 << 20  # DSPARK_STATIC_SCRATCH_BYTES of the C header
STATUS_NAMES = {0: "DSPARK_OK", 1: "DSPARK_ERR_INVALID_ARG", 2: "DSPARK_ERR_UNSUPPORTED",
                3: "DSPARK_ERR_CUDA", 4: "DSPARK_ERR_WORKSPACE"}
DTYPE_CODES = {torch.bfloat16: 0, torch.float32: 1}

SEQ_BAD_DRAFT = 1
SEQ_NONFINITE = 2
SEQ_ZERO_RESIDUAL = 4
SEQ_TIMEOUT = 8
SEQ_BAD_PARAM = 16


class DsparkError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


class AcceptOut(ctypes.Structure):
    _fields_ = [
        ("n_accepted", ctypes.c_void_p),
        ("tokens", ctypes.c_void_p),
        ("next_token", ctypes.c_void_p),
        ("status", ctypes.c_void_p),
        ("p_draft", ctypes.c_void_p),
        ("q_draft", ctypes.c_void_p),
        ("resid_mass", ctypes.c_void_p),
    ]


class Plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "elems_per_load", "loads_in_flight", "stream_threads_per_cta", "threads_per_cta",
        "chunk_elems", "n_chunks",
        "greedy_units_per_sequence", "sampling_units_per_sequence", "finish_ctas_per_sequence",
        "finish_threads_per_cta")]


QUENCH_MAX_WINDOW = 64  # DSPARK_QUENCH_MAX_WINDOW of include/dspark_policy.h
SPEC_ON, SPEC_OFF_YIELD, SPEC_OFF_KV = 0, 1, 2


class QuenchConfig(ctypes.Structure):
    _fields_ = [("break_even", ctypes.c_double), ("warmup", ctypes.c_int32),
                ("window", ctypes.c_int32), ("kv_limit", ctypes.c_int64)]


class QuenchState(ctypes.Structure):
    _fields_ = [("state", ctypes.c_int32), ("cycles", ctypes.c_int32),
                ("committed", ctypes.c_int64), ("window_sum", ctypes.c_int32),
                ("ring", ctypes.c_int32 * QUENCH_MAX_WINDOW)]


_LIB = None


def header_functions() -> list:
    """Names of every function declared in the headers under include/."""
    names = set()
    for h in sorted(os.listdir(build_lib.INCLUDE)):
        if h.endswith(".h"):
            text = open(os.path.join(build_lib.INCLUDE, h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(dspark_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def library_path() -> str:
    return build_lib.LIB_PATH


def load_library(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load (building first if needed) the CUDA library and declare its signatures."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = build_lib.LIB_PATH
    if not os.path.exists(path):
        if not build_if_missing:
            raise RuntimeError(f"CUDA library not built: {path}")
        build_lib.build()
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.dspark_status_string.restype = ctypes.c_char_p
    lib.dspark_status_string.argtypes = [i32]
    lib.dspark_version.restype = i32
    lib.dspark_version.argtypes = []
    lib.dspark_workspace_bytes.restype = sz
    lib.dspark_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.dspark_workspace_zero_bytes.restype = sz
    lib.dspark_workspace_zero_bytes.argtypes = [i32, i32]
    lib.dspark_plan.restype = i32
    lib.dspark_plan.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(Plan)]
    lib.dspark_greedy_accept.restype = i32
    lib.dspark_greedy_accept.argtypes = [vp, i64, vp, i64, i32, vp, i32, i32, i32, AcceptOut,
                                         vp, sz, vp]
    lib.dspark_speculative_sample_accept.restype = i32
    lib.dspark_speculative_sample_accept.argtypes = [vp, i64, vp, i64, vp, i32, vp, i32, i32,
                                                     i32, ctypes.c_float, vp, AcceptOut, vp, sz,
                                                     vp]
    lib.dspark_mixed_accept.restype = i32
    lib.dspark_mixed_accept.argtypes = [vp, i64, vp, i64, vp, i32, vp, vp, i32, i32, i32, vp, vp,
                                        AcceptOut, vp, sz, vp]
    lib.dspark_sample_pass1.restype = i32
    lib.dspark_sample_pass1.argtypes = [vp, i64, vp, i64, vp, i32, vp, i32, i32, i32,
                                        ctypes.c_float, vp, sz, vp]
    lib.dspark_early_exit_accept.restype = i32
    lib.dspark_early_exit_accept.argtypes = [vp, i64, vp, i64, vp, i32, vp, i32, i32, i32,
                                             ctypes.c_float, vp, AcceptOut, vp, sz, vp]
    lib.dspark_markov_matvec.restype = i32
    lib.dspark_markov_matvec.argtypes = [vp, i32, i32, i32, vp, i32, vp, vp]
    lib.dspark_markov_matvec_withheld.restype = i32
    lib.dspark_markov_matvec_withheld.argtypes = [vp, i32, i32, i32, vp, i32, vp, vp]
    lib.dspark_pipeline_timeouts.restype = i32
    lib.dspark_pipeline_timeouts.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)]
    lib.dspark_quench_reset.restype = i32
    lib.dspark_quench_reset.argtypes = [vp, i32]
    lib.dspark_quench_update.restype = i32
    lib.dspark_quench_update.argtypes = [ctypes.POINTER(QuenchConfig), vp, i32, vp, vp, vp]
    lib.dspark_speculative_sample_accept_static.restype = i32
    lib.dspark_speculative_sample_accept_static.argtypes = [vp, i64, vp, i64, vp, i32, vp, i32,
                                                            i32, i32, ctypes.c_float, vp,
                                                            AcceptOut, vp]
    _LIB = lib
    return lib


@dataclass
class AcceptResult:
    """Per-sequence result of one verify call (device tensors)."""

    n_accepted: torch.Tensor           # [B] int32: accepted drafts j (the host's n_keep)
    tokens: torch.Tensor               # [B, K+1] int32: x_0..x_{j-1}, token, then -1
    next_token: torch.Tensor           # [B] int32: correction (j < K) or bonus (j == K)
    status: torch.Tensor               # [B] int32 SEQ_* bits
    p_draft: Optional[torch.Tensor] = None     # [B, K] float32 p_i(x_i) (sampling)
    q_draft: Optional[torch.Tensor] = None     # [B, K] float32 q_i(x_i) (sampling)
    resid_mass: Optional[torch.Tensor] = None  # [B] float32 residual mass Z_j or 1 (sampling)

    @property
    def n_committed(self) -> torch.Tensor:
        """Tokens committed by the cycle: accepted drafts plus the correction / bonus."""
        return torch.where(self.next_token >= 0, self.n_accepted + 1, 0)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _split_block(P) -> Tuple[torch.Tensor, Optional[torch.Tensor], int, int]:
    """(p1, pv, ld_p1, ld_pv) in elements from a [B, K+1, V] block or a (p1, pv) pair."""
    if isinstance(P, (tuple, list)):
        p1, pv = P
        if p1.dim() != 2 or p1.stride(1) != 1:
            raise ValueError("p1 must be [B, V] with unit stride along V")
        if pv is not None and pv.shape[1] > 0:
            if pv.dim() != 3 or pv.stride(2) != 1 or pv.stride(1) != pv.shape[2]:
                raise ValueError("pv must be [B, K, V] with rows V apart")
            if pv.dtype != p1.dtype or pv.device != p1.device or pv.shape[0] != p1.shape[0] \
                    or pv.shape[2] != p1.shape[1]:
                raise ValueError("p1 and pv disagree in dtype, device or shape")
            return p1, pv, p1.stride(0), pv.stride(0)
        return p1, None, p1.stride(0), 0
    if P.dim() != 3 or P.stride(2) != 1 or P.stride(1) != P.shape[2]:
        raise ValueError("P must be [B, K+1, V] with rows V apart")
    K = P.shape[1] - 1
    return P[:, 0], (P[:, 1:] if K > 0 else None), P.stride(0), P.stride(0)


class _Workspace:
    """A per-device byte buffer reused across calls, grown on demand.

    The library needs the first ``dspark_workspace_zero_bytes(B, K)`` bytes (one counter per
    sequence) zero before a call, and a call leaves exactly its own such prefix zero; the bytes
    after it hold that call's other data. So the prefix is cleared again (a memset on the
    current stream; nothing is allocated) whenever a call needs more of it than the previous
    call left zero.
    """

    def __init__(self):
        self.bufs = {}
        self.zeroed = {}

    def get(self, device: torch.device, nbytes: int, B: int, K: int) -> torch.Tensor:
        key = device.index if device.index is not None else torch.cuda.current_device()
        need = int(load_library().dspark_workspace_zero_bytes(B, K))
        buf = self.bufs.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = new_workspace(max(nbytes, 256), device)
            self.bufs[key] = buf
        elif need > self.zeroed.get(key, 0):
            buf[:need].zero_()
        self.zeroed[key] = need
        return buf


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed workspace buffer of `nbytes` bytes (256-byte aligned, as every CUDA
    allocation): the state the library requires before its first call."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


_WS = _Workspace()


def workspace_bytes(B: int, K: int, V: int, dtype: torch.dtype) -> int:
    return int(load_library().dspark_workspace_bytes(B, K, V, DTYPE_CODES[dtype]))


def plan(B: int, K: int, V: int, dtype: torch.dtype, aligned16: bool = True) -> dict:
    p = Plan()
    rc = load_library().dspark_plan(B, K, V, DTYPE_CODES[dtype], int(aligned16), ctypes.byref(p))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_plan")
    return {n: getattr(p, n) for n, _ in Plan._fields_}


def _alloc_result(B: int, K: int, device, diagnostics: bool) -> AcceptResult:
    i32 = dict(dtype=torch.int32, device=device)
    res = AcceptResult(torch.empty(B, **i32), torch.empty(B, K + 1, **i32),
                       torch.empty(B, **i32), torch.empty(B, **i32))
    if diagnostics:
        res.p_draft = torch.empty(B, K, dtype=torch.float32, device=device)
        res.q_draft = torch.empty(B, K, dtype=torch.float32, device=device)
        res.resid_mass = torch.empty(B, dtype=torch.float32, device=device)
    return res


def _out_struct(r: AcceptResult) -> AcceptOut:
    return AcceptOut(_ptr(r.n_accepted), _ptr(r.tokens), _ptr(r.next_token), _ptr(r.status),
                     _ptr(r.p_draft), _ptr(r.q_draft), _ptr(r.resid_mass))


def _stream_handle(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def greedy_accept(P: Union[torch.Tensor, Tuple[torch.Tensor, torch.Tensor]],
                  drafts: torch.Tensor, *, out: Optional[AcceptResult] = None,
                  workspace: Optional[torch.Tensor] = None) -> AcceptResult:
    """Greedy block verify on the GPU: accept drafts while they equal the base argmax.

    ``workspace``, if given, is a device byte buffer of at least ``workspace_bytes(...)``
    bytes that no other call uses at the same time, whose first
    ``dspark_workspace_zero_bytes(B, K)`` bytes are zero (``new_workspace`` returns such a
    buffer; a call leaves its own prefix zero, so only a call with a larger B needs a clear).
    The current kernels need no zero prefix (the size is 0); the contract is kept general.
    """
    lib = load_library()
    p1, pv, ld_p1, ld_pv = _split_block(P)
    if not p1.is_cuda:
        raise RuntimeError("greedy_accept runs on CUDA tensors only")
    B, V = p1.shape
    K = 0 if pv is None else pv.shape[1]
    drafts = _check_drafts(drafts, B, K, p1.device)
    res = _check_out(out, B, K, p1.device) if out is not None else \
        _alloc_result(B, K, p1.device, diagnostics=False)
    nbytes = lib.dspark_workspace_bytes(B, K, V, DTYPE_CODES[p1.dtype])
    ws = workspace if workspace is not None else _WS.get(p1.device, nbytes, B, K)
    rc = lib.dspark_greedy_accept(_ptr(p1), ld_p1, _ptr(pv), ld_pv, DTYPE_CODES[p1.dtype],
                                  _ptr(drafts), B, K, V, _out_struct(res), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream_handle(p1.device))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_greedy_accept")
    return res


def speculative_sample_accept(P: Union[torch.Tensor, Tuple[torch.Tensor, torch.Tensor]],
                              Q: Optional[torch.Tensor], drafts: torch.Tensor,
                              temperature: float, uniforms: torch.Tensor, *,
                              out: Optional[AcceptResult] = None,
                              workspace: Optional[torch.Tensor] = None) -> AcceptResult:
    """Lossless rejection-sampling block verify on the GPU (T == 0 is greedy_accept)."""
    lib = load_library()
    p1, pv, ld_p1, ld_pv = _split_block(P)
    if not p1.is_cuda:
        raise RuntimeError("speculative_sample_accept runs on CUDA tensors only")
    B, V = p1.shape
    K = 0 if pv is None else pv.shape[1]
    drafts = _check_drafts(drafts, B, K, p1.device)
    if float(temperature) > 0:
        _check_sampling(Q, uniforms, p1, B, K, V)
    res = _check_out(out, B, K, p1.device) if out is not None else \
        _alloc_result(B, K, p1.device, diagnostics=True)
    nbytes = lib.dspark_workspace_bytes(B, K, V, DTYPE_CODES[p1.dtype])
    ws = workspace if workspace is not None else _WS.get(p1.device, nbytes, B, K)
    rc = lib.dspark_speculative_sample_accept(
        _ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), DTYPE_CODES[p1.dtype], _ptr(drafts), B, K,
        V, float(temperature), _ptr(uniforms), _out_struct(res), _ptr(ws),
        ws.numel() * ws.element_size(), _stream_handle(p1.device))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_speculative_sample_accept")
    return res


def mixed_accept(P: Union[torch.Tensor, Tuple[torch.Tensor, torch.Tensor]],
                 Q: Optional[torch.Tensor], drafts: torch.Tensor, temperatures: torch.Tensor,
                 uniforms: torch.Tensor, *, n_drafts: Optional[torch.Tensor] = None,
                 out: Optional[AcceptResult] = None,
                 workspace: Optional[torch.Tensor] = None) -> AcceptResult:
    """A mixed serving batch on the GPU: sequence b verifies its first n_drafts[b] drafts
    (all K when ``n_drafts`` is None) at temperatures[b], greedily where that is 0.

    ``temperatures`` is a float32 [B] tensor and ``n_drafts`` an int32 [B] tensor, both on
    P's device; u[b, n_drafts[b]] is sequence b's draw. Rows, drafts and uniforms past a
    sequence's count are never read. A bad count or temperature is reported per sequence
    (SEQ_BAD_PARAM).
    """
    lib = load_library()
    p1, pv, ld_p1, ld_pv = _split_block(P)
    if not p1.is_cuda:
        raise RuntimeError("mixed_accept runs on CUDA tensors only")
    B, V = p1.shape
    K = 0 if pv is None else pv.shape[1]
    drafts = _check_drafts(drafts, B, K, p1.device)
    if K > 0 and (Q is None or Q.shape != (B, K, V) or not Q.is_contiguous() or
                  Q.dtype != p1.dtype):
        raise ValueError("Q must be a contiguous [B, K, V] tensor of P's dtype")
    if uniforms.dtype != torch.float32 or uniforms.shape != (B, K + 1) or \
            not uniforms.is_contiguous() or uniforms.device != p1.device:
        raise ValueError("uniforms must be a contiguous float32 [B, K+1] tensor on P's device")
    if temperatures.dtype != torch.float32 or temperatures.shape != (B,) or \
            not temperatures.is_contiguous() or temperatures.device != p1.device:
        raise ValueError("temperatures must be a contiguous float32 [B] tensor on P's device")
    if n_drafts is not None and (n_drafts.dtype != torch.int32 or n_drafts.shape != (B,) or
                                 not n_drafts.is_contiguous() or n_drafts.device != p1.device):
        raise ValueError("n_drafts must be a contiguous int32 [B] tensor on P's device")
    res = _check_out(out, B, K, p1.device) if out is not None else \
        _alloc_result(B, K, p1.device, diagnostics=True)
    nbytes = lib.dspark_workspace_bytes(B, K, V, DTYPE_CODES[p1.dtype])
    ws = workspace if workspace is not None else _WS.get(p1.device, nbytes, B, K)
    rc = lib.dspark_mixed_accept(
        _ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), DTYPE_CODES[p1.dtype], _ptr(drafts),
        _ptr(n_drafts), B, K, V, _ptr(temperatures), _ptr(uniforms), _out_struct(res), _ptr(ws),
        ws.numel() * ws.element_size(), _stream_handle(p1.device))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_mixed_accept")
    return res


def early_exit_accept(P: Union[torch.Tensor, Tuple[torch.Tensor, torch.Tensor]],
                      Q: Optional[torch.Tensor], drafts: torch.Tensor, temperature: float,
                      uniforms: Optional[torch.Tensor], *, out: Optional[AcceptResult] = None,
                      workspace: Optional[torch.Tensor] = None) -> AcceptResult:
    """The verify step with early exit: each sequence's rows are read in draft order, in
    waves, until its first rejection (T == 0: its first greedy mismatch; Q and uniforms may
    then be None). Identical results to ``speculative_sample_accept`` on blocks whose rows
    are all usable; rows after a sequence's stop are never read."""
    lib = load_library()
    p1, pv, ld_p1, ld_pv = _split_block(P)
    if not p1.is_cuda:
        raise RuntimeError("early_exit_accept runs on CUDA tensors only")
    B, V = p1.shape
    K = 0 if pv is None else pv.shape[1]
    drafts = _check_drafts(drafts, B, K, p1.device)
    if temperature > 0:
        if K > 0 and (Q is None or Q.shape != (B, K, V) or not Q.is_contiguous() or
                      Q.dtype != p1.dtype):
            raise ValueError("Q must be a contiguous [B, K, V] tensor of P's dtype")
        if uniforms is None or uniforms.dtype != torch.float32 or \
                uniforms.shape != (B, K + 1) or not uniforms.is_contiguous() or \
                uniforms.device != p1.device:
            raise ValueError("uniforms must be a contiguous float32 [B, K+1] tensor on P's "
                             "device")
    res = _check_out(out, B, K, p1.device) if out is not None else \
        _alloc_result(B, K, p1.device, diagnostics=True)
    nbytes = lib.dspark_workspace_bytes(B, K, V, DTYPE_CODES[p1.dtype])
    ws = workspace if workspace is not None else _WS.get(p1.device, nbytes, B, K)
    rc = lib.dspark_early_exit_accept(
        _ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), DTYPE_CODES[p1.dtype], _ptr(drafts), B, K,
        V, float(temperature), _ptr(uniforms), _out_struct(res), _ptr(ws),
        ws.numel() * ws.element_size(), _stream_handle(p1.device))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_early_exit_accept")
    return res


MARKOV_TABLE_CODES = {"f16": 0, "q8_0": 1}


def markov_matvec(table: torch.Tensor, fmt: str, h: torch.Tensor, *,
                  out: Optional[torch.Tensor] = None, _withhold: bool = False) -> torch.Tensor:
    """The drafter's Markov-head table mat-vec on the GPU: y[b, v] = sum_k W[v, k] h[b, k].

    ``table`` holds markov_w2 as the drafter files store it: fmt "f16", a [V, R] float16 (or
    16-bit integer bits) tensor; fmt "q8_0", a [V, R/32 * 34] uint8 tensor of GGUF Q8_0 rows.
    ``h`` is a float32 [B, R] tensor on the same device (R = 256). Returns float32 [B, V].
    """
    lib = load_library()
    if fmt not in MARKOV_TABLE_CODES:
        raise ValueError("fmt must be 'f16' or 'q8_0'")
    if not table.is_cuda or not table.is_contiguous():
        raise ValueError("table must be a contiguous CUDA tensor")
    if h.dtype != torch.float32 or h.dim() != 2 or not h.is_contiguous() or \
            h.device != table.device:
        raise ValueError("h must be a contiguous float32 [B, R] tensor on the table's device")
    B, R = h.shape
    V = table.shape[0]
    row_bytes = R * 2 if fmt == "f16" else R // 32 * 34
    if table.dim() != 2 or table.shape[1] * table.element_size() != row_bytes:
        raise ValueError(f"table rows must be {row_bytes} bytes for fmt {fmt!r} and R = {R}")
    y = out if out is not None else torch.empty(B, V, dtype=torch.float32, device=h.device)
    if y.shape != (B, V) or y.dtype != torch.float32 or not y.is_contiguous():
        raise ValueError("out must be a contiguous float32 [B, V] tensor")
    fn = lib.dspark_markov_matvec_withheld if _withhold else lib.dspark_markov_matvec
    rc = fn(_ptr(table), MARKOV_TABLE_CODES[fmt], V, R, _ptr(h), B, _ptr(y),
            _stream_handle(h.device))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_markov_matvec")
    return y


def markov_matvec_withheld(table: torch.Tensor, fmt: str, h: torch.Tensor, *,
                           out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """markov_matvec with the first table copy of every CTA withheld, for tests of the timeout
    path only: the pipelined kernels' waits run out (about a second), they give up, and
    ``pipeline_timeouts()`` grows; the result is incomplete."""
    return markov_matvec(table, fmt, h, out=out, _withhold=True)


def pipeline_timeouts(device=None) -> int:
    """Waits inside the library's pipelined kernels that ran out on ``device`` (default: the
    current CUDA device) since the library was loaded; 0 unless a kernel gave up."""
    lib = load_library()
    n = ctypes.c_ulonglong(0)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        rc = lib.dspark_pipeline_timeouts(ctypes.byref(n))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_pipeline_timeouts")
    return int(n.value)


def speculative_sample_accept_static(P: Union[torch.Tensor, Tuple[torch.Tensor, torch.Tensor]],
                                     Q: Optional[torch.Tensor], drafts: torch.Tensor,
                                     temperature: float, uniforms: torch.Tensor, *,
                                     out: AcceptResult) -> AcceptResult:
    """speculative_sample_accept on the library's fixed per-device scratch: no workspace.

    ``out`` is required, so that the call itself allocates nothing. Shapes whose workspace
    exceeds STATIC_SCRATCH_BYTES raise DsparkError(DSPARK_ERR_WORKSPACE). Calls on one
    device that overlap on the GPU share the scratch and race.
    """
    lib = load_library()
    p1, pv, ld_p1, ld_pv = _split_block(P)
    B, V = p1.shape
    K = 0 if pv is None else pv.shape[1]
    # every layout check before anything reaches the library: it checks pointers for null,
    # not the sizes behind them
    drafts = _check_drafts(drafts, B, K, p1.device)
    if float(temperature) > 0:
        _check_sampling(Q, uniforms, p1, B, K, V)
    if out is None:
        raise ValueError("out is required: the call allocates nothing")
    _check_out(out, B, K, p1.device)
    if not p1.is_cuda:
        raise RuntimeError("speculative_sample_accept_static runs on CUDA tensors only")
    # the library resolves its scratch on the current device: make it P's
    with torch.cuda.device(p1.device):
        rc = lib.dspark_speculative_sample_accept_static(
            _ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), DTYPE_CODES[p1.dtype], _ptr(drafts), B,
            K, V, float(temperature), _ptr(uniforms), _out_struct(out),
            _stream_handle(p1.device))
    if rc != DSPARK_OK:
        raise DsparkError(rc, "dspark_speculative_sample_accept_static")
    return out


def _check_sampling(Q: Optional[torch.Tensor], uniforms: torch.Tensor, p1: torch.Tensor, B: int,
                    K: int, V: int) -> None:
    """Q [B, K, V] contiguous in P's dtype on P's device (K > 0), uniforms float32 [B, K+1]."""
    if K > 0:
        if Q is None or Q.shape != (B, K, V) or not Q.is_contiguous() or Q.dtype != p1.dtype \
                or Q.device != p1.device:
            raise ValueError("Q must be a contiguous [B, K, V] tensor of P's dtype and device")
    if uniforms is None or uniforms.dtype != torch.float32 or uniforms.shape != (B, K + 1) or \
            not uniforms.is_contiguous() or uniforms.device != p1.device:
        raise ValueError("uniforms must be a contiguous float32 [B, K+1] tensor on P's device")


_OUT_SHAPES = {"n_accepted": (torch.int32, 1), "tokens": (torch.int32, 2),
               "next_token": (torch.int32, 1), "status": (torch.int32, 1),
               "p_draft": (torch.float32, 2), "q_draft": (torch.float32, 2),
               "resid_mass": (torch.float32, 1)}


def _check_out(out: AcceptResult, B: int, K: int, device) -> AcceptResult:
    """A caller-supplied result: every tensor it holds is contiguous, on P's device, of its
    field's dtype and shape (the kernels write B, B x (K+1) or B x K elements there)."""
    shapes = {1: (B,), 2: (B, K)}
    for name, (dtype, rank) in _OUT_SHAPES.items():
        t = getattr(out, name)
        if t is None:
            if name in ("n_accepted", "tokens", "next_token"):
                raise ValueError(f"out.{name} is required")
            continue
        shape = (B, K + 1) if name == "tokens" else shapes[rank]
        if t.dtype != dtype or tuple(t.shape) != shape or not t.is_contiguous() or \
                t.device != device:
            raise ValueError(f"out.{name} must be a contiguous {dtype} tensor of shape "
                             f"{list(shape)} on P's device")
    return out


def _check_drafts(drafts: Optional[torch.Tensor], B: int, K: int, device) -> Optional[torch.Tensor]:
    if K == 0:
        return drafts
    if drafts.dtype != torch.int32 or drafts.shape != (B, K) or not drafts.is_contiguous() \
            or drafts.device != device:
        raise ValueError("drafts must be a contiguous int32 [B, K] tensor on P's device")
    return drafts


class PreparedCall:
    """A verify call with its arguments marshalled once, for tight timing loops.

    Holds references to every tensor it points at. Calling it enqueues the same kernels as
    the corresponding function above on the stream captured at construction.
    """

    def __init__(self, policy: str, P, Q, drafts, temperature, uniforms, out: AcceptResult,
                 workspace: torch.Tensor, n_drafts: Optional[torch.Tensor] = None):
        self.lib = load_library()
        p1, pv, ld_p1, ld_pv = _split_block(P)
        B, V = p1.shape
        K = 0 if pv is None else pv.shape[1]
        self.keep = (P, Q, drafts, uniforms, out, workspace, p1, pv, temperature, n_drafts)
        dt = DTYPE_CODES[p1.dtype]
        stream = _stream_handle(p1.device)
        nbytes = workspace.numel() * workspace.element_size()
        if policy == "greedy":
            self.fn = self.lib.dspark_greedy_accept
            self.args = (_ptr(p1), ld_p1, _ptr(pv), ld_pv, dt, _ptr(drafts), B, K, V,
                         _out_struct(out), _ptr(workspace), nbytes, stream)
        elif policy == "sample_pass1":  # the sampling call's pass 1 alone (timing)
            self.fn = self.lib.dspark_sample_pass1
            self.args = (_ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), dt, _ptr(drafts), B, K, V,
                         float(temperature), _ptr(workspace), nbytes, stream)
        elif policy == "early_exit":
            self.fn = self.lib.dspark_early_exit_accept
            self.args = (_ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), dt, _ptr(drafts), B, K, V,
                         float(temperature), _ptr(uniforms), _out_struct(out), _ptr(workspace),
                         nbytes, stream)
        elif policy == "mixed":  # temperature: float32 [B] tensor
            self.fn = self.lib.dspark_mixed_accept
            self.args = (_ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), dt, _ptr(drafts),
                         _ptr(n_drafts), B, K, V, _ptr(temperature), _ptr(uniforms),
                         _out_struct(out), _ptr(workspace), nbytes, stream)
        else:
            self.fn = self.lib.dspark_speculative_sample_accept
            self.args = (_ptr(p1), ld_p1, _ptr(pv), ld_pv, _ptr(Q), dt, _ptr(drafts), B, K, V,
                         float(temperature), _ptr(uniforms), _out_struct(out), _ptr(workspace),
                         nbytes, stream)
        self.name = policy

    def __call__(self):
        rc = self.fn(*self.args)
        if rc != DSPARK_OK:
            raise DsparkError(rc, self.name)


class YieldQuench:
    """The yield-quench speculation policy over a batch of requests (include/dspark_policy.h).

    After each verify step, ``update`` takes every request's ``n_accepted`` (a negative value:
    not verified this step) and, optionally, its context depth, and returns which requests
    should keep drafting: a request stops for good once the mean committed tokens of its last
    ``window`` cycles fall below ``break_even`` (after ``warmup`` cycles), or once its context
    exceeds ``kv_limit`` tokens (the DeepSeek-V4-Flash DSpark drafter card's 64k gate). The
    controller runs in the C library on host arrays.
    """

    def __init__(self, n_requests: int, break_even: float, warmup: int = 8, window: int = 16,
                 kv_limit: int = 65536):
        self.lib = load_library()
        self.config = QuenchConfig(float(break_even), int(warmup), int(window), int(kv_limit))
        self.n = int(n_requests)
        self.states = (QuenchState * max(1, self.n))()
        rc = self.lib.dspark_quench_reset(ctypes.cast(self.states, ctypes.c_void_p), self.n)
        if rc != DSPARK_OK:
            raise DsparkError(rc, "dspark_quench_reset")

    def update(self, n_accepted, kv_depth=None):
        import numpy as np

        na = np.ascontiguousarray(
            n_accepted.cpu().numpy() if isinstance(n_accepted, torch.Tensor) else n_accepted,
            dtype=np.int32)
        if na.shape != (self.n,):
            raise ValueError(f"n_accepted must have shape [{self.n}]")
        kv = None
        if kv_depth is not None:
            kv = np.ascontiguousarray(
                kv_depth.cpu().numpy() if isinstance(kv_depth, torch.Tensor) else kv_depth,
                dtype=np.int64)
            if kv.shape != (self.n,):
                raise ValueError(f"kv_depth must have shape [{self.n}]")
        out = np.zeros(self.n, dtype=np.int32)
        rc = self.lib.dspark_quench_update(
            ctypes.byref(self.config), ctypes.cast(self.states, ctypes.c_void_p), self.n,
            na.ctypes.data, None if kv is None else kv.ctypes.data, out.ctypes.data)
        if rc != DSPARK_OK:
            raise DsparkError(rc, "dspark_quench_update")
        return out.astype(bool)

    def state(self, b: int) -> dict:
        s = self.states[b]
        return {"state": s.state, "cycles": s.cycles, "committed": s.committed,
                "window_sum": s.window_sum}
