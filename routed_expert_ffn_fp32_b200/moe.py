"""ctypes binding of libmoe_b200.so (include/moe.h), argument marshalling only.

Every function has the C entry point's name and takes torch tensors where the
C function takes device pointers; PyTorch only provides device memory and
streams.  A non-zero status raises MoeError.  Every computation runs in the
library's CUDA kernels: there is no fallback, and loading fails loudly when
the library has not been built.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_DEVICE_DATA = -6

MOE_PATH_AUTO = 0
MOE_PATH_GEMV = 1
MOE_PATH_GEMM = 2

MOE_ACT_EXACT = 0
MOE_ACT_MXFP4 = 1

MOE_DEBUG_STARVE_FIRST_WAIT = 1

#: every symbol include/moe.h declares
EXPORTS = (
    "moe_workspace_bytes", "moe_workspace_init", "moe_route_topk", "moe_bucket",
    "moe_expert_ffn_mxfp4", "moe_combine", "moe_layer_forward", "moe_act_quant_mxfp4",
    "moe_decode_mxfp4", "moe_get_error", "moe_status_string", "moe_version",
    "moe_layer_forward_static", "moe_get_error_static", "moe_workspace_set_limits",
    "moe_combine_range", "moe_round_bf16",
    "moe_slot_bank_bytes", "moe_slot_bank_create", "moe_slot_bank_destroy", "moe_slot_bank_acquire",
    "moe_slot_bank_experts", "moe_slot_bank_stats", "moe_layer_forward_banked",
    "moe_layer_forward_banked_workspace_bytes",
)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


class moe_shape_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32)]


class moe_mxfp4_experts_t(ctypes.Structure):
    _fields_ = [("gate_q", ctypes.c_void_p), ("gate_s", ctypes.c_void_p),
                ("up_q", ctypes.c_void_p), ("up_s", ctypes.c_void_p),
                ("down_q", ctypes.c_void_p), ("down_s", ctypes.c_void_p),
                ("n_experts", ctypes.c_int32)]


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libmoe_b200.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m routed_expert_ffn_fp32_b200.build` "
            "(there is no non-CUDA implementation)")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    shape = moe_shape_t
    ex = ctypes.POINTER(moe_mxfp4_experts_t)
    sig = {
        "moe_workspace_bytes": (sz, [shape, i32, i32, i32]),
        "moe_workspace_init": (i32, [vp, sz, vp]),
        "moe_route_topk": (i32, [vp, vp, vp, shape, vp, vp, vp, vp, sz, vp]),
        "moe_bucket": (i32, [vp, shape, vp, vp, vp, vp, sz, vp]),
        "moe_expert_ffn_mxfp4": (i32, [ex, ex, vp, vp, vp, shape, i32, i32, vp, vp, sz, vp]),
        "moe_combine": (i32, [vp, vp, shape, i32, vp, vp]),
        "moe_combine_range": (i32, [vp, vp, vp, i32, i32, shape, i32, vp, vp]),
        "moe_round_bf16": (i32, [vp, ctypes.c_int64, vp, vp]),
        "moe_slot_bank_bytes": (sz, [i32, i32, i32]),
        "moe_slot_bank_create": (i32, [ex, i32, i32, i32, vp, sz, ctypes.POINTER(vp)]),
        "moe_slot_bank_destroy": (None, [vp]),
        "moe_slot_bank_acquire": (i32, [vp, vp, i32, vp, vp]),
        "moe_slot_bank_experts": (i32, [vp, ex]),
        "moe_slot_bank_stats": (i32, [vp, ctypes.POINTER(ctypes.c_int64),
                                      ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)]),
        "moe_layer_forward_banked": (i32, [vp, vp, vp, vp, ex, shape, i32, i32, vp, vp, vp, vp, sz, vp]),
        "moe_layer_forward_banked_workspace_bytes": (sz, [shape, i32, i32, i32, i32]),
        "moe_layer_forward": (i32, [vp, vp, vp, ex, ex, shape, i32, i32, vp, vp, vp, vp, sz, vp]),
        "moe_layer_forward_static": (i32, [vp, vp, vp, ex, ex, shape, i32, vp, vp, vp, vp]),
        "moe_act_quant_mxfp4": (i32, [vp, i32, i32, vp, vp, vp]),
        "moe_decode_mxfp4": (i32, [vp, vp, i32, i32, vp, vp]),
        "moe_get_error": (i32, [vp, vp]),
        "moe_get_error_static": (i32, [vp]),
        "moe_workspace_set_limits": (i32, [vp, ctypes.c_uint32, ctypes.c_uint32, vp]),
        "moe_status_string": (ctypes.c_char_p, [i32]),
        "moe_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


# ---------------------------------------------------------------- helpers ---
def _p(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _s(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def status_string(status: int) -> str:
    return load_library().moe_status_string(status).decode()


def shape_of(T: int, H: int, I: int, E: int, k: int) -> moe_shape_t:
    return moe_shape_t(T, H, I, E, k)


@dataclasses.dataclass
class Experts:
    """Device tensors of n MXFP4 experts in the library's layout."""
    gate_q: torch.Tensor
    gate_s: torch.Tensor
    up_q: torch.Tensor
    up_s: torch.Tensor
    down_q: torch.Tensor
    down_s: torch.Tensor

    @property
    def n_experts(self) -> int:
        return int(self.gate_q.shape[0])

    def cstruct(self) -> moe_mxfp4_experts_t:
        return moe_mxfp4_experts_t(_p(self.gate_q), _p(self.gate_s), _p(self.up_q), _p(self.up_s),
                                   _p(self.down_q), _p(self.down_s), self.n_experts)

    @classmethod
    def from_numpy(cls, d: dict, device="cuda") -> "Experts":
        return cls(**{n: torch.from_numpy(d[n]).to(device) for n in
                      ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")})

    def nbytes(self) -> int:
        return sum(t.numel() for t in (self.gate_q, self.gate_s, self.up_q, self.up_s,
                                       self.down_q, self.down_s))


def _ex(e):
    return None if e is None else ctypes.byref(e.cstruct())


# --------------------------------------------------------------- C entries ---
def moe_workspace_bytes(shape: moe_shape_t, path: int = MOE_PATH_AUTO,
                        precision: int = MOE_ACT_EXACT, has_shared: bool = False) -> int:
    return int(load_library().moe_workspace_bytes(shape, path, precision, int(has_shared)))


def moe_workspace_init(ws: torch.Tensor, stream=None):
    _check(load_library().moe_workspace_init(_p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "moe_workspace_init")


def make_workspace(shape: moe_shape_t, path=MOE_PATH_AUTO, precision=MOE_ACT_EXACT,
                   has_shared=False, device="cuda", stream=None) -> torch.Tensor:
    n = moe_workspace_bytes(shape, path, precision, has_shared)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream)
    return ws


def moe_route_topk(x, w_router, bias, shape, topk_idx, topk_w, ws, logits_out=None, stream=None):
    _check(load_library().moe_route_topk(_p(x), _p(w_router), _p(bias), shape, _p(logits_out),
                                         _p(topk_idx), _p(topk_w), _p(ws), ws.numel(), _s(stream)),
           "moe_route_topk")


def moe_bucket(topk_idx, shape, counts, offsets, entries, ws, stream=None):
    _check(load_library().moe_bucket(_p(topk_idx), shape, _p(counts), _p(offsets), _p(entries),
                                     _p(ws), ws.numel(), _s(stream)), "moe_bucket")


def moe_expert_ffn_mxfp4(experts: Experts, shared, x, offsets, entries, shape, partial_out, ws,
                         path=MOE_PATH_AUTO, precision=MOE_ACT_EXACT, stream=None):
    _check(load_library().moe_expert_ffn_mxfp4(_ex(experts), _ex(shared), _p(x), _p(offsets),
                                               _p(entries), shape, path, precision,
                                               _p(partial_out), _p(ws), ws.numel(), _s(stream)),
           "moe_expert_ffn_mxfp4")


def moe_combine(partial, topk_w, shape, has_shared, y, stream=None):
    _check(load_library().moe_combine(_p(partial), _p(topk_w), shape, int(has_shared), _p(y),
                                      _s(stream)), "moe_combine")


def moe_combine_range(partial, topk_w, topk_idx, e_begin, e_end, shape, has_shared, y_f32,
                      stream=None):
    _check(load_library().moe_combine_range(_p(partial), _p(topk_w), _p(topk_idx), e_begin, e_end,
                                            shape, int(has_shared), _p(y_f32), _s(stream)),
           "moe_combine_range")


def moe_round_bf16(x_f32, out, stream=None):
    _check(load_library().moe_round_bf16(_p(x_f32), x_f32.numel(), _p(out), _s(stream)),
           "moe_round_bf16")


class SlotBank:
    """Routed experts in pinned host memory, n_slots of them resident in a
    device slot bank (moe_slot_bank_*).  ``host`` holds CPU tensors in the
    library's layout; they are pinned here if they are not already."""

    def __init__(self, host: "Experts", H: int, I: int, n_slots: int, device="cuda"):
        lib = load_library()
        self.host = Experts(**{f: (t if t.is_pinned() else t.pin_memory())
                               for f, t in dataclasses.asdict(host).items()})
        n = int(lib.moe_slot_bank_bytes(H, I, n_slots))
        if n == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_slot_bank_bytes")
        self.mem = torch.empty(n, dtype=torch.uint8, device=device)
        self.n_slots = n_slots
        h = self.host
        hs = moe_mxfp4_experts_t(h.gate_q.data_ptr(), h.gate_s.data_ptr(), h.up_q.data_ptr(),
                                 h.up_s.data_ptr(), h.down_q.data_ptr(), h.down_s.data_ptr(),
                                 int(h.gate_q.shape[0]))
        self._h = ctypes.c_void_p()
        _check(lib.moe_slot_bank_create(ctypes.byref(hs), H, I, n_slots, self.mem.data_ptr(), n,
                                        ctypes.byref(self._h)), "moe_slot_bank_create")

    @property
    def handle(self):
        return self._h

    def acquire(self, ids, stream=None):
        """Make experts ``ids`` (ints) resident; returns their slots."""
        arr = (ctypes.c_int32 * len(ids))(*ids)
        out = (ctypes.c_int32 * len(ids))()
        _check(load_library().moe_slot_bank_acquire(self._h, arr, len(ids), out, _s(stream)),
               "moe_slot_bank_acquire")
        return list(out)

    def stats(self):
        h, m, e = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(load_library().moe_slot_bank_stats(self._h, ctypes.byref(h), ctypes.byref(m),
                                                  ctypes.byref(e)), "moe_slot_bank_stats")
        return h.value, m.value, e.value

    def close(self):
        if self._h:
            load_library().moe_slot_bank_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_layer_forward_banked(x, w_router, bias, bank: SlotBank, shared, shape, y, ws, topk_idx,
                             topk_w, path=MOE_PATH_AUTO, precision=MOE_ACT_EXACT, stream=None):
    """The layer over a slot bank: routes, reads the chosen experts back once
    (one synchronisation of the stream), makes them resident and runs the
    FFNs over the bank's slots.  topk_idx / topk_w receive the routing."""
    _check(load_library().moe_layer_forward_banked(_p(x), _p(w_router), _p(bias), bank.handle,
                                                   _ex(shared), shape, path, precision, _p(y),
                                                   _p(topk_idx), _p(topk_w), _p(ws), ws.numel(),
                                                   _s(stream)), "moe_layer_forward_banked")


def banked_workspace(shape, n_slots, path=MOE_PATH_AUTO, precision=MOE_ACT_EXACT,
                     has_shared=False, device="cuda", stream=None) -> torch.Tensor:
    """A zeroed workspace for moe_layer_forward_banked with n_slots slots."""
    n = int(load_library().moe_layer_forward_banked_workspace_bytes(shape, n_slots, path, precision,
                                                                    int(has_shared)))
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_layer_forward_banked_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream)
    return ws


def moe_layer_forward(x, w_router, bias, experts: Experts, shared, shape, y, ws,
                      path=MOE_PATH_AUTO, precision=MOE_ACT_EXACT, topk_idx=None, topk_w=None,
                      stream=None):
    _check(load_library().moe_layer_forward(_p(x), _p(w_router), _p(bias), _ex(experts),
                                            _ex(shared), shape, path, precision, _p(y),
                                            _p(topk_idx), _p(topk_w), _p(ws), ws.numel(),
                                            _s(stream)), "moe_layer_forward")


def moe_layer_forward_static(x, w_router, bias, experts: Experts, shared, shape, y,
                             precision=MOE_ACT_EXACT, topk_idx=None, topk_w=None, stream=None):
    """moe_layer_forward without a workspace: the library's own fixed scratch
    array stands in for it (for callers that may not allocate)."""
    _check(load_library().moe_layer_forward_static(_p(x), _p(w_router), _p(bias), _ex(experts),
                                                   _ex(shared), shape, precision, _p(y),
                                                   _p(topk_idx), _p(topk_w), _s(stream)),
           "moe_layer_forward_static")


def moe_act_quant_mxfp4(inp, q_out, s_out, stream=None):
    rows, K = inp.shape
    _check(load_library().moe_act_quant_mxfp4(_p(inp), rows, K, _p(q_out), _p(s_out), _s(stream)),
           "moe_act_quant_mxfp4")


def moe_decode_mxfp4(q, s, K, out, stream=None):
    rows = q.shape[0]
    _check(load_library().moe_decode_mxfp4(_p(q), _p(s), rows, K, _p(out), _s(stream)),
           "moe_decode_mxfp4")


def moe_get_error(ws, stream=None) -> int:
    return int(load_library().moe_get_error(_p(ws), _s(stream)))


def moe_get_error_static(stream=None) -> int:
    return int(load_library().moe_get_error_static(_s(stream)))


def moe_workspace_set_limits(ws, wait_us: int = 0, debug: int = 0, stream=None):
    _check(load_library().moe_workspace_set_limits(_p(ws), wait_us, debug, _s(stream)),
           "moe_workspace_set_limits")


def moe_version() -> str:
    return load_library().moe_version().decode()
