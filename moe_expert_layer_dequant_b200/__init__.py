"""Python binding of libmoeffn.so, the B200 quantized gated FFN / MoE layer library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch provides device memory and streams. The functions keep the
names of the C ABI (include/moeffn.h):

* ``ffn_dense``          -- dense gated FFN + raw residual add (in place)
* ``ffn_shared_expert``  -- Gemma-style shared expert + post-FFN RMSNorm
* ``moe_router_topk``    -- router GEMV, top-k softmax, grouped pair order
* ``MoePlan`` / ``moe_layer`` -- routed MoE layer with a seeded rank-ordered
  sum and a raw residual add (in place)
* ``ffn_dense_prenorm`` / ``moe_layer_prenorm`` -- the same layers with their
  input RMSNorm (m = rms_norm(residual, w)) applied inside the library

There is no CPU fallback: importing this package fails if the library is
missing, and every call raises ``MoeffnError`` on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoeffn.so")

# moeffn_qformat / moeffn_act / moeffn_kind
Q_INT8_ROW, Q_INT4_AFFINE_G32, BF16, F32, Q_Q4_K = 1, 2, 3, 4, 5
ACT_SILU, ACT_GELU_TANH = 0, 1
KIND_DENSE, KIND_SHARED, KIND_ROUTER, KIND_MOE = 1, 2, 3, 4
ACTS = {"silu": ACT_SILU, "gelu_tanh": ACT_GELU_TANH}
FORMATS = {"int8_row": Q_INT8_ROW, "int4_g32": Q_INT4_AFFINE_G32, "q4_k": Q_Q4_K}


class MoeffnError(RuntimeError):
    """A library call returned a non-zero moeffn_status."""

    def __init__(self, status: int, message: str):
        super().__init__(f"moeffn status {status}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libmoeffn.so is not built ({LIB_PATH}); run python moe_expert_layer_dequant_b200/build.py")
_lib = ctypes.CDLL(LIB_PATH)


class _QWeight(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int32), ("rows", ctypes.c_int32), ("cols", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("min", ctypes.c_void_p)]


class _FFN(ctypes.Structure):
    _fields_ = [("gate", _QWeight), ("up", _QWeight), ("down", _QWeight)]


class _MoeDesc(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("act", ctypes.c_int32),
                ("router", _QWeight), ("experts", ctypes.POINTER(_FFN)), ("shared", ctypes.POINTER(_FFN)),
                ("shared_gate", ctypes.POINTER(_QWeight)), ("expert_scale", ctypes.c_void_p),
                ("shared_post_norm", ctypes.c_void_p), ("shared_post_norm_eps", ctypes.c_float)]


_vp, _sz, _i, _f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_SIGS = {
    "moeffn_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moeffn_last_error": (ctypes.c_char_p, []),
    "ffn_dense": (_i, [ctypes.POINTER(_FFN), _vp, _vp, _i, _i, _vp, _sz, _vp]),
    "ffn_dense_noalloc": (_i, [ctypes.POINTER(_FFN), _vp, _vp, _i, _i, _vp]),
    "ffn_dense_prenorm": (_i, [ctypes.POINTER(_FFN), _vp, _f, _vp, _i, _i, _vp, _sz, _vp]),
    "moe_layer_prenorm": (_i, [_vp, _vp, _f, _vp, _i, _vp, _vp, _sz, _vp]),
    "ffn_shared_expert": (_i, [ctypes.POINTER(_FFN), _vp, _vp, _f, _vp, _i, _i, _vp, _sz, _vp]),
    "moe_router_topk": (_i, [ctypes.POINTER(_QWeight), _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_plan_create": (_i, [ctypes.POINTER(_MoeDesc), ctypes.POINTER(_vp)]),
    "moe_plan_destroy": (_i, [_vp]),
    "moe_workspace_bytes": (_sz, [_vp, _i]),
    "moe_layer": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _sz, _vp]),
    "moeffn_test_dequant": (_i, [ctypes.POINTER(_QWeight), _vp, _vp, _vp]),
    "moeffn_profile_enable": (_i, [_i]),
    "moeffn_device_faults": (ctypes.c_uint, [_i]),
    "moeffn_profile_read": (_i, [ctypes.c_char_p, _i, _vp, _vp, _i, ctypes.POINTER(_i)]),
    "moeffn_test_topk_from_logits": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moeffn_test_inject_gemv_fault": (_i, [_i, _i, ctypes.c_uint]),
    "moe_dispatch_rows": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_experts_workspace_bytes": (_sz, [_vp, _i]),
    "moe_experts_grouped": (_i, [_vp, _vp, _i, _vp, _i, _vp, _vp, _sz, _vp]),
    "moe_combine_workspace_bytes": (_sz, [_i, _i]),
    "moe_combine": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def _check(status: int) -> None:
    if status != 0:
        raise MoeffnError(status, _lib.moeffn_last_error().decode())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ----------------------------------------------------------------------------- weights


@dataclass
class QWeight:
    """A quantized (or plain) matrix in device memory, W[rows][cols].

    The C struct handed to the library is built on the first call and reused
    while every field's device pointer and element count stay the same; a new
    tensor in a field, or a tensor whose storage moved (``set_``, ``resize_``),
    rebuilds it."""
    format: int
    rows: int
    cols: int
    q: torch.Tensor
    scale: Optional[torch.Tensor] = None
    min: Optional[torch.Tensor] = None
    _cache: tuple = field(default=(None, None), init=False, repr=False, compare=False)

    def _key(self) -> tuple:
        def k(t):
            return None if t is None else (t.data_ptr(), t.numel())
        return (self.format, self.rows, self.cols, k(self.q), k(self.scale), k(self.min))

    def c(self) -> _QWeight:
        """The C struct, built once and rebuilt when a field is reassigned."""
        key = self._key()
        if self._cache[0] != key:
            self._cache = (key, _QWeight(self.format, self.rows, self.cols, _ptr(self.q), _ptr(self.scale),
                                         _ptr(self.min)))
        return self._cache[1]

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.q, self.scale, self.min) if t is not None)


@dataclass
class FFN:
    gate: QWeight
    up: QWeight
    down: QWeight

    _cache: tuple = field(default=(None, None), init=False, repr=False, compare=False)

    def c(self) -> _FFN:
        """The C struct, built once and rebuilt when a matrix or one of its fields changes."""
        key = (self.gate._key(), self.up._key(), self.down._key())
        if self._cache[0] != key:
            self._cache = (key, _FFN(self.gate.c(), self.up.c(), self.down.c()))
        return self._cache[1]

    @property
    def nbytes(self) -> int:
        return self.gate.nbytes + self.up.nbytes + self.down.nbytes


def qweight_from_arrays(fmt: str, rows: int, cols: int, q, scale=None, mn=None, device="cuda") -> QWeight:
    """Upload numpy storage arrays (codes, fp16 scale, fp16 min) as a QWeight."""
    def up(a):
        if a is None:
            return None
        return torch.from_numpy(a.copy()).to(device)
    return QWeight(FORMATS[fmt], rows, cols, up(q), up(scale), up(mn))


def upload_qweight(w, device="cuda") -> QWeight:
    """Upload a host matrix object with fields fmt, N, K, q, scale, min (numpy)."""
    return qweight_from_arrays(w.fmt, w.N, w.K, w.q, w.scale, w.min, device)


def upload_ffn(f, device="cuda") -> FFN:
    """Upload a host FFN object with fields gate, up, down (see upload_qweight)."""
    return FFN(upload_qweight(f.gate, device), upload_qweight(f.up, device), upload_qweight(f.down, device))


def plain_weight(t: torch.Tensor) -> QWeight:
    """A plain bf16 or fp32 [rows][cols] device matrix (router, gate vector)."""
    fmt = BF16 if t.dtype in (torch.bfloat16, torch.int16, torch.uint16) else F32
    if t.dtype == torch.float32:
        fmt = F32
    rows, cols = (1, t.shape[0]) if t.dim() == 1 else t.shape
    return QWeight(fmt, int(rows), int(cols), t)


# ----------------------------------------------------------------------------- workspace


def workspace_bytes(kind: int, M: int, H: int, I: int, E: int = 0, top_k: int = 0) -> int:
    return int(_lib.moeffn_workspace_bytes(kind, M, H, I, E, top_k))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device buffer of at least nbytes (torch's allocator aligns to 512)."""
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def _ws(ws: Optional[torch.Tensor], need):
    """(workspace, pointer, bytes); `need()` sizes one when the caller gave none
    (a given workspace is checked by the library itself)."""
    if ws is None:
        ws = alloc_workspace(need())
    return ws, _ptr(ws), ws.numel()


# ----------------------------------------------------------------------------- calls


def ffn_dense(w: FFN, x: torch.Tensor, residual: torch.Tensor, act: str = "silu",
              ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """residual <- bf16(residual + bf16(FFN(x))); x, residual bf16 [M][H]."""
    M, H = x.shape
    ws, wp, wn = _ws(ws, lambda: workspace_bytes(KIND_DENSE, M, H, w.gate.rows))
    f = w.c()
    _check(_lib.ffn_dense(ctypes.byref(f), _ptr(x), _ptr(residual), M, ACTS[act], wp, wn, _stream(stream)))
    return residual


def ffn_dense_prenorm(w: FFN, norm_w: torch.Tensor, residual: torch.Tensor, act: str = "silu", eps: float = 1e-6,
                      ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """residual <- bf16(residual + bf16(FFN(rms_norm(residual, norm_w)))); the input norm runs in the library."""
    M, H = residual.shape
    ws, wp, wn = _ws(ws, lambda: workspace_bytes(KIND_DENSE, M, H, w.gate.rows))
    f = w.c()
    _check(_lib.ffn_dense_prenorm(ctypes.byref(f), _ptr(norm_w), float(eps), _ptr(residual), M, ACTS[act], wp, wn,
                                  _stream(stream)))
    return residual


NOALLOC_SCRATCH_BYTES = 4 << 20


def ffn_dense_noalloc(w: FFN, x: torch.Tensor, residual: torch.Tensor, act: str = "silu", stream=None) -> torch.Tensor:
    """ffn_dense with the library's fixed scratch array instead of a workspace.

    For callers that cannot allocate device memory when they call; the call
    allocates nothing. Raises MoeffnError (status -3) when the call needs more
    than NOALLOC_SCRATCH_BYTES of scratch. All calls share one array, so calls
    that may overlap on the GPU must be serialized by the caller.
    """
    M = x.shape[0]
    f = w.c()
    _check(_lib.ffn_dense_noalloc(ctypes.byref(f), _ptr(x), _ptr(residual), M, ACTS[act], _stream(stream)))
    return residual


def ffn_shared_expert(w: FFN, x: torch.Tensor, norm_w: torch.Tensor, h1_out: torch.Tensor, act: str = "gelu_tanh",
                      eps: float = 1e-6, ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """h1_out <- RMSNorm(bf16(FFN(x))) * norm_w; all bf16."""
    M, H = x.shape
    ws, wp, wn = _ws(ws, lambda: workspace_bytes(KIND_SHARED, M, H, w.gate.rows))
    f = w.c()
    _check(_lib.ffn_shared_expert(ctypes.byref(f), _ptr(x), _ptr(norm_w), float(eps), _ptr(h1_out), M, ACTS[act],
                                  wp, wn, _stream(stream)))
    return h1_out


def moe_router_topk(router: QWeight, x: torch.Tensor, top_k: int, logits_out=None, perm=None, expert_offsets=None,
                    ws: Optional[torch.Tensor] = None, stream=None):
    """Returns (topk_idx int32 [M][k], topk_w float32 [M][k]); fills the optional outputs."""
    M, H = x.shape
    idx = torch.empty((M, top_k), dtype=torch.int32, device=x.device)
    w = torch.empty((M, top_k), dtype=torch.float32, device=x.device)
    ws, wp, wn = _ws(ws, lambda: workspace_bytes(KIND_ROUTER, M, H, 0, router.rows, top_k))
    r = router.c()
    _check(_lib.moe_router_topk(ctypes.byref(r), _ptr(x), M, top_k, _ptr(logits_out), _ptr(idx), _ptr(w),
                                _ptr(perm), _ptr(expert_offsets), wp, wn, _stream(stream)))
    return idx, w


class MoePlan:
    """A routed MoE layer: router, E expert FFNs (INT4-affine), optional shared expert.

    Qwen form (default): the shared expert is gated by sigmoid(shared_gate . x)
    and seeds the routed sum. Gemma form (``shared_post_norm`` given): the
    shared branch is normed (post-FFN RMSNorm, ``shared_post_norm_eps``) and
    joins in the tail; ``expert_scale`` (fp32 [E]) scales the routing weights.
    """

    def __init__(self, router: QWeight, experts: Sequence[FFN], top_k: int, act: str = "silu",
                 shared: Optional[FFN] = None, shared_gate: Optional[QWeight] = None,
                 expert_scale: Optional[torch.Tensor] = None, shared_post_norm: Optional[torch.Tensor] = None,
                 shared_post_norm_eps: float = 1e-6):
        self.router, self.experts, self.shared, self.shared_gate = router, list(experts), shared, shared_gate
        self.expert_scale, self.shared_post_norm = expert_scale, shared_post_norm
        self.top_k, self.E, self.H = top_k, len(experts), router.cols
        arr = (_FFN * len(experts))(*[e.c() for e in experts])
        self._keep = [arr]
        desc = _MoeDesc(len(experts), top_k, ACTS[act], router.c(), arr, None, None,
                        _ptr(expert_scale), _ptr(shared_post_norm), float(shared_post_norm_eps))
        if shared is not None:
            sf = _FFN(shared.gate.c(), shared.up.c(), shared.down.c())
            self._keep.append(sf)
            desc.shared = ctypes.pointer(sf)
        if shared_gate is not None:
            sg = shared_gate.c()
            self._keep.append(sg)
            desc.shared_gate = ctypes.pointer(sg)
        h = ctypes.c_void_p()
        _check(_lib.moe_plan_create(ctypes.byref(desc), ctypes.byref(h)))
        self._h = h

    def workspace_bytes(self, M: int) -> int:
        return int(_lib.moe_workspace_bytes(self._h, M))

    def close(self):
        if getattr(self, "_h", None):
            _lib.moe_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_layer(plan: MoePlan, x: torch.Tensor, residual: torch.Tensor, topk_idx_out: Optional[torch.Tensor] = None,
              ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """residual <- bf16(residual + bf16(seeded rank-ordered routed sum)); bf16 [M][H]."""
    M = x.shape[0]
    ws, wp, wn = _ws(ws, lambda: plan.workspace_bytes(M))
    _check(_lib.moe_layer(plan._h, _ptr(x), _ptr(residual), M, _ptr(topk_idx_out), wp, wn, _stream(stream)))
    return residual


def moe_layer_prenorm(plan: MoePlan, norm_w: torch.Tensor, residual: torch.Tensor, eps: float = 1e-6,
                      topk_idx_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """moe_layer on m = rms_norm(residual, norm_w), formed inside the library."""
    M = residual.shape[0]
    ws, wp, wn = _ws(ws, lambda: plan.workspace_bytes(M))
    _check(_lib.moe_layer_prenorm(plan._h, _ptr(norm_w), float(eps), _ptr(residual), M, _ptr(topk_idx_out), wp, wn,
                                  _stream(stream)))
    return residual


def device_faults(clear: bool = True) -> int:
    """Fault word of the kernels' bounded waits (0: none); blocking."""
    return int(_lib.moeffn_device_faults(1 if clear else 0))


def profile_enable(on: bool = True) -> None:
    """Bracket each library kernel launch with CUDA events (see moeffn_profile_read)."""
    _check(_lib.moeffn_profile_enable(1 if on else 0))


def profile_read(max_kernels: int = 64) -> dict:
    """{kernel name: (launches, total device ms)} since the previous read."""
    names = ctypes.create_string_buffer(4096)
    counts = (ctypes.c_int32 * max_kernels)()
    ms = (ctypes.c_float * max_kernels)()
    n = ctypes.c_int(0)
    _check(_lib.moeffn_profile_read(names, 4096, ctypes.addressof(counts), ctypes.addressof(ms), max_kernels,
                                    ctypes.byref(n)))
    keys = names.value.decode().split("\n")[: n.value]
    return {k: (int(counts[i]), float(ms[i])) for i, k in enumerate(keys)}


def test_dequant(w: QWeight, want_f32=True, want_bf16=True, stream=None):
    """Device dequantization of W (test export): (fp32 [N][K] or None, bf16 bits [N][K] or None)."""
    dev = w.q.device
    f = torch.empty((w.rows, w.cols), dtype=torch.float32, device=dev) if want_f32 else None
    b = torch.empty((w.rows, w.cols), dtype=torch.int16, device=dev) if want_bf16 else None
    c = w.c()
    _check(_lib.moeffn_test_dequant(ctypes.byref(c), _ptr(f), _ptr(b), _stream(stream)))
    return f, b


def test_inject_gemv_fault(kind: int, value: int = 0, wait_us: int = 2000) -> None:
    """One-shot failure injection into the next dense gate/up GEMV launch (test export):
    kind 1 stops its producer at stage `value` (bounded waits of `wait_us` run out,
    fault bit 0), kind 2 forces ring depth `value` (refused by the kernel, fault bit 1),
    kind 0 cancels."""
    _check(_lib.moeffn_test_inject_gemv_fault(kind, value, wait_us))


def test_topk_from_logits(logits: torch.Tensor, top_k: int, stream=None):
    """Top-k / weights / grouped order from given fp32 logits (test export)."""
    M, E = logits.shape
    dev = logits.device
    idx = torch.empty((M, top_k), dtype=torch.int32, device=dev)
    w = torch.empty((M, top_k), dtype=torch.float32, device=dev)
    perm = torch.empty(M * top_k, dtype=torch.int32, device=dev)
    offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    uni = torch.empty(E, dtype=torch.int32, device=dev)
    nu = torch.empty(1, dtype=torch.int32, device=dev)
    _check(_lib.moeffn_test_topk_from_logits(_ptr(logits), M, E, top_k, _ptr(idx), _ptr(w), _ptr(perm), _ptr(offs),
                                             _ptr(uni), _ptr(nu), _stream(stream)))
    return idx, w, perm, offs, uni[: int(nu.item())]


__all__ = ["ffn_dense", "ffn_dense_prenorm", "moe_layer_prenorm", "ffn_dense_noalloc", "ffn_shared_expert", "moe_router_topk", "moe_layer", "MoePlan", "QWeight", "FFN",
           "qweight_from_arrays", "upload_qweight", "upload_ffn", "plain_weight", "workspace_bytes", "alloc_workspace", "test_dequant",
           "test_topk_from_logits", "test_inject_gemv_fault", "profile_enable", "profile_read", "device_faults", "MoeffnError", "LIB_PATH"]


# ----------------------------------------------------------------------------- expert-parallel pieces


def moe_dispatch_rows(x: torch.Tensor, topk_idx: torch.Tensor, perm: torch.Tensor, top_k: int, stream=None):
    """Token rows of the M*k pair slots in perm's (expert) order and each slot's
    expert: returns (rows bf16 bits [M*k][H], experts int32 [M*k])."""
    M, H = x.shape
    P = M * top_k
    rows = torch.empty((P, H), dtype=x.dtype, device=x.device)
    experts = torch.empty(P, dtype=torch.int32, device=x.device)
    _check(_lib.moe_dispatch_rows(_ptr(x), _ptr(topk_idx), _ptr(perm), M, top_k, H, _ptr(rows), _ptr(experts),
                                  _stream(stream)))
    return rows, experts


def moe_experts_grouped(plan: MoePlan, rows: torch.Tensor, row_expert: torch.Tensor, expert_base: int = 0,
                        d_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Down outputs (fp32 [R][H]) of the plan's experts for rows in any order:
    row i goes through expert row_expert[i] - expert_base of the plan."""
    R, H = rows.shape
    if d_out is None:
        d_out = torch.empty((R, H), dtype=torch.float32, device=rows.device)
    if R == 0:
        return d_out
    ws, wp, wn = _ws(ws, lambda: int(_lib.moe_experts_workspace_bytes(plan._h, R)))
    _check(_lib.moe_experts_grouped(plan._h, _ptr(rows), R, _ptr(row_expert), int(expert_base), _ptr(d_out), wp, wn,
                                    _stream(stream)))
    return d_out


def moe_combine(d: torch.Tensor, perm: torch.Tensor, topk_w: torch.Tensor, residual: torch.Tensor,
                shared_d: Optional[torch.Tensor] = None, gate_logit: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """residual <- bf16(residual + bf16(seed + sum_r w_r d_{t,r})), d in perm's slot order (fp32 [M*k][H])."""
    M, H = residual.shape
    k = topk_w.shape[1]
    ws, wp, wn = _ws(ws, lambda: int(_lib.moe_combine_workspace_bytes(M, k)))
    _check(_lib.moe_combine(_ptr(d), _ptr(perm), _ptr(topk_w), M, k, H, _ptr(shared_d), _ptr(gate_logit),
                            _ptr(residual), wp, wn, _stream(stream)))
    return residual
