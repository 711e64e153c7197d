"""Thin Python binding of libcolimoe (include/coli_moe.h).

Every function here only marshals arguments to the C ABI function of the same
name; all computation on the device happens in the library's CUDA kernels.
Device buffers are torch CUDA tensors (PyTorch serves as the allocator and the
stream source); host buffers are numpy arrays.  Importing this package loads the
in-tree ``libcolimoe.so`` and raises if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "ColiError", "COLI_F32", "COLI_BF16", "COLI_PATH_AUTO", "COLI_PATH_GEMV",
    "COLI_PATH_GEMM", "COLI_PATH_FUSED", "COLI_PATH_TWOPASS", "lib", "EXPORTS",
    "coli_moe_last_error", "coli_moe_quantize", "coli_moe_expert_bytes",
    "coli_moe_pack_expert", "coli_moe_quantize_expert_device", "coli_moe_layer_create",
    "coli_moe_layer_destroy", "coli_moe_workspace_size", "coli_moe_route",
    "coli_moe_union", "coli_moe_forward", "coli_moe_forward_ex", "coli_moe_rmsnorm",
    "coli_moe_stack_workspace_size", "coli_moe_stack_forward", "coli_moe_dequant_debug",
    "coli_moe_forward_noalloc", "NOALLOC_SCRATCH_BYTES", "coli_moe_status", "Desc",
    "coli_moe_layer_set_topp", "coli_moe_layer_set_partition",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcolimoe.so")

COLI_F32, COLI_BF16 = 0, 1
COLI_PATH_AUTO, COLI_PATH_GEMV, COLI_PATH_GEMM, COLI_PATH_FUSED, COLI_PATH_TWOPASS = 0, 1, 2, 3, 4

# every symbol include/coli_moe.h declares
EXPORTS = (
    "coli_moe_last_error", "coli_moe_quantize", "coli_moe_expert_bytes",
    "coli_moe_pack_expert", "coli_moe_quantize_expert_device", "coli_moe_layer_create",
    "coli_moe_layer_destroy", "coli_moe_workspace_size", "coli_moe_route",
    "coli_moe_union", "coli_moe_forward", "coli_moe_forward_ex", "coli_moe_rmsnorm",
    "coli_moe_stack_workspace_size", "coli_moe_stack_forward", "coli_moe_dequant_debug",
    "coli_moe_forward_noalloc", "coli_moe_status", "coli_moe_host_workspace_size",
    "coli_moe_forward_host", "coli_moe_stack_host_workspace_size", "coli_moe_stack_forward_host",
    "coli_moe_quantize_expert_fp8_device", "coli_moe_quantize8", "coli_moe_expert_bytes8",
    "coli_moe_pack_expert8", "coli_moe_layer_set_topp", "coli_moe_layer_set_partition",
    "coli_moe_quantize_expert8_device", "coli_moe_layer_set_wait_test", "coli_moe_union_readback",
)


class ColiError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libcolimoe error {code}: {msg}")
        self.code = code


class Desc(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("group", ctypes.c_int32), ("routed_scale", ctypes.c_float),
                ("norm_topk", ctypes.c_int32), ("router_w", ctypes.c_void_p),
                ("router_b", ctypes.c_void_p), ("experts", ctypes.c_void_p),
                ("bits", ctypes.c_int32)]


from . import build as _build  # noqa: E402

if _build.stale():
    try:
        _build.build()
    except Exception as exc:  # no fallback: the CUDA library is the product
        raise ImportError(f"{LIB_PATH} is missing or stale and nvcc failed: {exc}") from exc

lib = ctypes.CDLL(LIB_PATH)

_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "coli_moe_last_error": ([], ctypes.c_char_p),
    "coli_moe_quantize": ([_P, _I64, _I64, _I32, _P, _P], ctypes.c_int),
    "coli_moe_expert_bytes": ([_I32, _I32, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "coli_moe_pack_expert": ([_I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "coli_moe_quantize_expert_device": ([_I32, _I32, _I32, _P, _P, _P, _P, _P], ctypes.c_int),
    "coli_moe_quantize_expert8_device": ([_I32, _I32, _I32, _P, _P, _P, _P, _P], ctypes.c_int),
    "coli_moe_quantize_expert_fp8_device": ([_I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P],
                                            ctypes.c_int),
    "coli_moe_quantize8": ([_P, _I64, _I64, _I32, _P, _P], ctypes.c_int),
    "coli_moe_expert_bytes8": ([_I32, _I32, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "coli_moe_pack_expert8": ([_I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "coli_moe_layer_create": ([ctypes.POINTER(Desc), ctypes.POINTER(_P)], ctypes.c_int),
    "coli_moe_layer_destroy": ([_P], ctypes.c_int),
    "coli_moe_layer_set_topp": ([_P, ctypes.c_float], ctypes.c_int),
    "coli_moe_layer_set_wait_test": ([_P, _I32], ctypes.c_int),
    "coli_moe_layer_set_partition": ([_P, _I32, _I32, _I32, _P], ctypes.c_int),
    "coli_moe_workspace_size": ([_P, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "coli_moe_route": ([_P, _P, ctypes.c_int, _I32, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "coli_moe_union": ([_P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "coli_moe_forward": ([_P, _P, ctypes.c_int, _I32, _P, _P, _SZ, _P], ctypes.c_int),
    "coli_moe_forward_ex": ([_P, _P, ctypes.c_int, _I32, _P, _P, ctypes.c_int, _P, _P, _P,
                             _P, _SZ, _P], ctypes.c_int),
    "coli_moe_rmsnorm": ([_P, _I32, _I32, ctypes.c_float, _P, _P], ctypes.c_int),
    "coli_moe_stack_workspace_size": ([_P, _I32, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "coli_moe_stack_forward": ([_P, _I32, _P, _I32, ctypes.c_float, ctypes.c_int, _P, _SZ,
                                _P], ctypes.c_int),
    "coli_moe_dequant_debug": ([_P, _I32, _I32, _P, _P], ctypes.c_int),
    "coli_moe_union_readback": ([_P, _I32, _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "coli_moe_forward_noalloc": ([_P, _P, ctypes.c_int, _I32, _P, _P], ctypes.c_int),
    "coli_moe_status": ([_P, _I32, _P, ctypes.POINTER(_I32), _P], ctypes.c_int),
    "coli_moe_host_workspace_size": ([_P, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "coli_moe_forward_host": ([_P, _P, ctypes.c_int, _I32, _P, ctypes.c_int, _P, _SZ, _P],
                              ctypes.c_int),
    "coli_moe_stack_host_workspace_size": ([_P, _I32, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "coli_moe_stack_forward_host": ([_P, _I32, _P, _P, _I32, ctypes.c_float, ctypes.c_int, _P,
                                     _SZ, _P], ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def coli_moe_last_error() -> str:
    return lib.coli_moe_last_error().decode()


def _ok(rc: int):
    if rc != 0:
        raise ColiError(rc, coli_moe_last_error())


def _ptr(a):
    """Device or host address of a torch tensor / numpy array / int / None."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data
    assert a.is_contiguous(), "tensors passed to libcolimoe must be contiguous"
    return a.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return s if isinstance(s, int) else s.cuda_stream


def _xtype(x):
    import torch
    if x.dtype == torch.float32:
        return COLI_F32
    if x.dtype == torch.bfloat16:
        return COLI_BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {x.dtype}")


# ---------------------------------------------------------------------------
def coli_moe_quantize(w: np.ndarray, group: int):
    """Host quantiser -> (packed uint8 [R, K/2], scales f32 [R, K/G])."""
    w = np.ascontiguousarray(w, np.float32)
    R, K = w.shape
    ng = 1 if group == 0 else max(K // group, 1)
    packed = np.zeros((R, K // 2), np.uint8)
    scales = np.zeros((R, ng), np.float32)
    _ok(lib.coli_moe_quantize(_ptr(w), R, K, group, _ptr(packed), _ptr(scales)))
    return packed, scales


def coli_moe_expert_bytes(H: int, I: int, group: int) -> int:
    out = _SZ()
    _ok(lib.coli_moe_expert_bytes(H, I, group, ctypes.byref(out)))
    return out.value


def coli_moe_pack_expert(H, I, group, gate_codes, gate_scales, up_codes, up_scales,
                         down_codes, down_scales) -> np.ndarray:
    blob = np.zeros((coli_moe_expert_bytes(H, I, group),), np.uint8)
    arrs = [np.ascontiguousarray(a) for a in
            (gate_codes, gate_scales, up_codes, up_scales, down_codes, down_scales)]
    _ok(lib.coli_moe_pack_expert(H, I, group, *[_ptr(a) for a in arrs], _ptr(blob)))
    return blob


def coli_moe_quantize8(w: np.ndarray, group: int):
    """Host 8-bit quantiser -> (codes int8 [R, K], scales f32 [R, K/G])."""
    w = np.ascontiguousarray(w, np.float32)
    R, K = w.shape
    ng = 1 if group == 0 else max(K // group, 1)
    codes = np.zeros((R, K), np.int8)
    scales = np.zeros((R, ng), np.float32)
    _ok(lib.coli_moe_quantize8(_ptr(w), R, K, group, _ptr(codes), _ptr(scales)))
    return codes, scales


def coli_moe_expert_bytes8(H: int, I: int, group: int) -> int:
    out = _SZ()
    _ok(lib.coli_moe_expert_bytes8(H, I, group, ctypes.byref(out)))
    return out.value


def coli_moe_pack_expert8(H, I, group, gate_codes, gate_scales, up_codes, up_scales,
                          down_codes, down_scales) -> np.ndarray:
    blob = np.zeros((coli_moe_expert_bytes8(H, I, group),), np.uint8)
    arrs = [np.ascontiguousarray(a) for a in
            (gate_codes, gate_scales, up_codes, up_scales, down_codes, down_scales)]
    _ok(lib.coli_moe_pack_expert8(H, I, group, *[_ptr(a) for a in arrs], _ptr(blob)))
    return blob


def coli_moe_quantize_expert_device(H, I, group, gate, up, down, blob, stream=None):
    _ok(lib.coli_moe_quantize_expert_device(H, I, group, _ptr(gate), _ptr(up), _ptr(down),
                                            _ptr(blob), _stream(stream)))


def coli_moe_quantize_expert8_device(H, I, group, gate, up, down, blob, stream=None):
    _ok(lib.coli_moe_quantize_expert8_device(H, I, group, _ptr(gate), _ptr(up), _ptr(down),
                                             _ptr(blob), _stream(stream)))


def coli_moe_quantize_expert_fp8_device(H, I, group, gate, up, down, gate_bs, up_bs, down_bs,
                                        blob, stream=None):
    """FP8 E4M3 codes (uint8 device tensors) with 128 x 128 block scales -> int4 blob."""
    _ok(lib.coli_moe_quantize_expert_fp8_device(H, I, group, _ptr(gate), _ptr(up), _ptr(down),
                                                _ptr(gate_bs), _ptr(up_bs), _ptr(down_bs),
                                                _ptr(blob), _stream(stream)))


def coli_moe_layer_create(desc: Desc) -> ctypes.c_void_p:
    h = _P()
    _ok(lib.coli_moe_layer_create(ctypes.byref(desc), ctypes.byref(h)))
    return h


def coli_moe_layer_destroy(layer) -> None:
    _ok(lib.coli_moe_layer_destroy(layer))


def coli_moe_layer_set_wait_test(layer, withhold_stage: int) -> None:
    """Test only: make the fused kernel's bounded waits run out (see the header)."""
    _ok(lib.coli_moe_layer_set_wait_test(layer, withhold_stage))


def coli_moe_layer_set_topp(layer, p: float) -> None:
    _ok(lib.coli_moe_layer_set_topp(layer, p))


def coli_moe_layer_set_partition(layer, e_begin: int, e_end: int, with_shared: bool,
                                 experts) -> None:
    _ok(lib.coli_moe_layer_set_partition(layer, e_begin, e_end, int(bool(with_shared)),
                                         _ptr(experts)))


def coli_moe_workspace_size(layer, T: int) -> int:
    out = _SZ()
    _ok(lib.coli_moe_workspace_size(layer, T, ctypes.byref(out)))
    return out.value


def coli_moe_route(layer, x, T, idx, w, ws, stream=None):
    _ok(lib.coli_moe_route(layer, _ptr(x), _xtype(x), T, _ptr(idx), _ptr(w), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream)))


def coli_moe_union(idx, T, k, E, offsets, pair_tok, pair_slot, uniq, n_uniq, stream=None):
    _ok(lib.coli_moe_union(_ptr(idx), T, k, E, _ptr(offsets), _ptr(pair_tok),
                           _ptr(pair_slot), _ptr(uniq), _ptr(n_uniq), _stream(stream)))


def coli_moe_forward(layer, x, T, y, ws, stream=None):
    _ok(lib.coli_moe_forward(layer, _ptr(x), _xtype(x), T, _ptr(y), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)))


COLI_STAGES = 5
STAGE_NAMES = ("router", "union", "gateup", "down", "combine")


def coli_moe_forward_ex(layer, x, T, y, ws, residual=None, path=COLI_PATH_AUTO, idx_out=None,
                        w_out=None, events=None, stream=None):
    """events: None or COLI_STAGES + 1 torch.cuda.Event(enable_timing=True)."""
    ev = None
    if events is not None:
        assert len(events) == COLI_STAGES + 1
        for e in events:          # torch creates the CUDA event on its first record
            if not e.cuda_event:
                e.record()
        ev = (_P * len(events))(*[e.cuda_event for e in events])
    _ok(lib.coli_moe_forward_ex(layer, _ptr(x), _xtype(x), T, _ptr(y), _ptr(residual), path,
                                _ptr(idx_out), _ptr(w_out), ev, _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)))


def coli_moe_rmsnorm(x, T, H, eps, out, stream=None):
    _ok(lib.coli_moe_rmsnorm(_ptr(x), T, H, eps, _ptr(out), _stream(stream)))


def _layer_array(layers):
    arr = (_P * len(layers))(*[l.value if isinstance(l, _P) else l for l in layers])
    return arr


def coli_moe_stack_workspace_size(layers, T: int) -> int:
    out = _SZ()
    _ok(lib.coli_moe_stack_workspace_size(_layer_array(layers), len(layers), T,
                                          ctypes.byref(out)))
    return out.value


def coli_moe_stack_forward(layers, x, T, eps, ws, path=COLI_PATH_AUTO, stream=None):
    _ok(lib.coli_moe_stack_forward(_layer_array(layers), len(layers), _ptr(x), T, eps, path,
                                   _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def coli_moe_host_workspace_size(layer, T: int) -> int:
    out = _SZ()
    _ok(lib.coli_moe_host_workspace_size(layer, T, ctypes.byref(out)))
    return out.value


def coli_moe_forward_host(layer, x_host, T, y_host, ws, path=COLI_PATH_AUTO, stream=None):
    """x_host / y_host: host tensors (page-locked for graph capture); ws on the device."""
    _ok(lib.coli_moe_forward_host(layer, _ptr(x_host), _xtype(x_host), T, _ptr(y_host), path,
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def coli_moe_stack_host_workspace_size(layers, T: int) -> int:
    out = _SZ()
    _ok(lib.coli_moe_stack_host_workspace_size(_layer_array(layers), len(layers), T,
                                               ctypes.byref(out)))
    return out.value


def coli_moe_stack_forward_host(layers, x_host, y_host, T, eps, ws, path=COLI_PATH_AUTO,
                                stream=None):
    _ok(lib.coli_moe_stack_forward_host(_layer_array(layers), len(layers), _ptr(x_host),
                                        _ptr(y_host), T, eps, path, _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)))


def coli_moe_status(layer, T: int, ws, stream=None) -> int:
    """Error flags of the last forward on this workspace (raises on a timeout);
    ws None: the built-in scratch array of coli_moe_forward_noalloc."""
    flags = _I32(0)
    _ok(lib.coli_moe_status(layer, T, _ptr(ws), ctypes.byref(flags), _stream(stream)))
    return flags.value


def coli_moe_union_readback(layer, T: int, ws, offsets=None, pair_tok=None, pair_slot=None,
                            uniq=None, n_uniq=None, inv=None, stream=None):
    """Test helper: the union the last forward on ws built (see the header)."""
    _ok(lib.coli_moe_union_readback(layer, T, _ptr(ws), _ptr(offsets), _ptr(pair_tok),
                                    _ptr(pair_slot), _ptr(uniq), _ptr(n_uniq), _ptr(inv),
                                    _stream(stream)))


def coli_moe_dequant_debug(layer, expert: int, which: int, out, stream=None):
    _ok(lib.coli_moe_dequant_debug(layer, expert, which, _ptr(out), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 8 << 20  # COLI_NOALLOC_SCRATCH_BYTES in include/coli_moe.h


def coli_moe_forward_noalloc(layer, x, T, y, stream=None):
    """Forward without a caller workspace, for hosts that cannot allocate device
    memory: the library's built-in scratch array is used instead (see the header
    for its limit and for the rule that overlapping calls must be serialised)."""
    _ok(lib.coli_moe_forward_noalloc(layer, _ptr(x), _xtype(x), T, _ptr(y), _stream(stream)))
