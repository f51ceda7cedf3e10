"""Thin ctypes binding over libmoe.so (include/moe_w4a16.h).

Argument marshalling only: tensors are passed as device pointers and the
current torch stream is passed as the cudaStream_t; every step of the layer
runs in libmoe's CUDA kernels.  Importing this module loads the library and
raises ImportError if it has not been built (there is no fallback path).
"""
import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moe_w4a16.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'`")

lib = ctypes.CDLL(LIB_PATH)

FMT_INT4_G128, FMT_NVFP4, FMT_BF16 = 0, 1, 2
STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_CUDA",
          -4: "MOE_ERR_TIMEOUT", -5: "MOE_ERR_WORKSPACE", -6: "MOE_ERR_DEVICE_INDEX", -7: "MOE_ERR_NONFINITE"}

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t


class QWeight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("num_experts", ctypes.c_int32), ("out_dim", ctypes.c_int32),
                ("in_dim", ctypes.c_int32), ("packed", _P), ("scales", _P), ("global_scale", _P),
                ("input_scale", _P)]


class Layer(ctypes.Structure):
    _fields_ = [("gate", QWeight), ("up", QWeight), ("down", QWeight),
                ("sh_gate", QWeight), ("sh_up", QWeight), ("sh_down", QWeight),
                ("router_w", _P), ("router_bias", _P),
                ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("F", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("swiglu_limit", ctypes.c_float), ("act_f16", ctypes.c_int32)]


def _sig(name, res, args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("moe_workspace_bytes", _SZ, [_I, _I, _I, _I, _I])
_sig("moe_workspace_init", _I, [_P, _SZ, _P])
_sig("moe_read_status", _I, [_P, _P, ctypes.POINTER(ctypes.c_int32)])
_sig("moe_set_wait_limit", _I, [_P, ctypes.c_uint64, _P])
_sig("moe_set_wait_hold", _I, [_P, _I, _P])
_sig("moe_status_string", ctypes.c_char_p, [_I])
_sig("moe_launch_count", ctypes.c_uint64, [])
_sig("moe_route_topk", _I, [_P, _I, _I, _P, _P, _I, _I, _P, _P, _P, _SZ, _P])
_sig("moe_permute", _I, [_P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P])
_sig("moe_permute_noalloc", _I, [_P, _I, _I, _I, _P, _P, _P, _P])
_sig("moe_grouped_w4a16_swiglu", _I, [_P, _I, _I, _P, _P, _I, _P, _P, _F, _P, _P, _SZ, _P])
_sig("moe_grouped_w4a16_down", _I, [_P, _P, _P, _P, _I, _P, _P, _P, _SZ, _P])
_sig("moe_unpermute_combine", _I, [_P, _P, _I, _I, _I, _P, _P, _P])
_sig("moe_layer_decode", _I, [_P, _I, _P, _P, _P, _SZ, _P])
_sig("moe_layer_forward", _I, [_P, _I, _P, _P, _P, _SZ, _P])
_sig("moe_layer_graph_create", _I, [_P, _I, _P, _P, _P, _SZ, ctypes.POINTER(_P)])
_sig("moe_layer_graph_launch", _I, [_P, _P])
_sig("moe_layer_graph_destroy", _I, [_P])
_sig("moe_quantize_int4_g128", _I, [_P, _I64, _I64, _P, _P, _P])
_sig("moe_quantize_nvfp4", _I, [_P, _I64, _I64, _P, _P, _P, _P, _SZ, _P])
_sig("moe_quantize_nvfp4_act", _I, [_P, _I64, _I64, _P, _P, _P, _P])
_sig("moe_csf_decode", _I, [_P, _P, _P, _I, _I, _I, _P, _P, _P])
_sig("moe_csf_encode_workspace_bytes", _SZ, [_I, _I])
_sig("moe_csf_encode", _I, [_P, _I, _I, _I, _P, _P, _P, _I64, _P, _SZ, _P])


def declared_functions():
    """Names of the functions declared in the public header."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|uint64_t|const char\*)\s+(moe_\w+)\s*\(", text, flags=re.M)))


class MoEError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({lib.moe_status_string(code).decode()})")
        self.code = code


def _check(fn, code):
    if code != 0:
        raise MoEError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


class Bank:
    """A projection bank in the fused layout [E, out, in] (device tensors).

    int4:  packed int32 [E,out,in/8], scales bf16 [E,out,in/128]
    nvfp4: packed uint8 [E,out,in/2], scales uint8 [E,out,in/16], global_scale fp32 [E]
    bf16:  packed bf16 [E,out,in]
    """

    def __init__(self, fmt, packed, scales=None, global_scale=None, out_dim=None, in_dim=None, input_scale=None):
        self.fmt, self.packed, self.scales, self.global_scale = fmt, packed, scales, global_scale
        self.input_scale = input_scale       # NVFP4 W4A4: activation global scale by expert, fp32 [E]
        self.E = packed.shape[0]
        self.out_dim = packed.shape[1] if out_dim is None else out_dim
        mult = {FMT_INT4_G128: 8, FMT_NVFP4: 2, FMT_BF16: 1}[fmt]
        self.in_dim = packed.shape[2] * mult if in_dim is None else in_dim

    def struct(self):
        return QWeight(self.fmt, self.E, self.out_dim, self.in_dim, _ptr(self.packed),
                       _ptr(self.scales), _ptr(self.global_scale), _ptr(self.input_scale))


def _empty_qweight():
    return QWeight(0, 0, 0, 0, None, None, None, None)


class MoELayer:
    def __init__(self, gate, up, down, router_w, top_k=8, router_bias=None, shared=None, act_f16=False):
        self.act_f16 = act_f16               # x and y in fp16 instead of bf16
        self.gate, self.up, self.down = gate, up, down
        self.shared = shared
        self.router_w, self.router_bias = router_w, router_bias
        self.E, self.H = router_w.shape
        self.F = gate.out_dim
        self.top_k = top_k

    def struct(self):
        sh = self.shared
        return Layer(self.gate.struct(), self.up.struct(), self.down.struct(),
                     sh[0].struct() if sh else _empty_qweight(),
                     sh[1].struct() if sh else _empty_qweight(),
                     sh[2].struct() if sh else _empty_qweight(),
                     _ptr(self.router_w), _ptr(self.router_bias),
                     self.E, self.H, self.F, self.top_k, 0.0, 1 if self.act_f16 else 0)


def workspace_bytes(T, H, E, F, top_k):
    return int(lib.moe_workspace_bytes(T, H, E, F, top_k))


def workspace(T, H, E, F, top_k, device="cuda"):
    n = workspace_bytes(T, H, E, F, top_k)
    if n == 0:
        raise MoEError("moe_workspace_bytes", -2)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check("moe_workspace_init", lib.moe_workspace_init(_ptr(ws), n, _stream()))
    return ws


def launch_count():
    """Kernels the library has launched in this process so far."""
    return int(lib.moe_launch_count())


def read_status(ws):
    v = ctypes.c_int32(0)
    _check("moe_read_status", lib.moe_read_status(_ptr(ws), _stream(), ctypes.byref(v)))
    return int(v.value)


def set_wait_limit(ws, limit_ns):
    """Bound on each device wait of the kernels using this workspace (0 = default)."""
    _check("moe_set_wait_limit", lib.moe_set_wait_limit(_ptr(ws), int(limit_ns), _stream()))


def set_wait_hold(ws, hold):
    """Failure testing: the tensor-core GEMMs using this workspace first wait on a barrier nothing completes."""
    _check("moe_set_wait_hold", lib.moe_set_wait_hold(_ptr(ws), int(bool(hold)), _stream()))


def route_topk(x, router_w, router_bias, top_k, ws):
    T, H = x.shape
    E = router_w.shape[0]
    ids = torch.empty(T, top_k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, top_k, dtype=torch.float32, device=x.device)
    _check("moe_route_topk", lib.moe_route_topk(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, top_k,
                                                _ptr(ids), _ptr(w), _ptr(ws), ws.numel(), _stream()))
    return ids, w


def permute(ids, E, ws):
    T, k = ids.shape
    off = torch.empty(E + 1, dtype=torch.int32, device=ids.device)
    rs = torch.empty(T * k, dtype=torch.int32, device=ids.device)
    sr = torch.empty(T * k, dtype=torch.int32, device=ids.device)
    _check("moe_permute", lib.moe_permute(_ptr(ids), T, k, E, _ptr(off), _ptr(rs), _ptr(sr),
                                          _ptr(ws), ws.numel(), _stream()))
    return off, rs, sr


def permute_noalloc(ids, E):
    """moe_permute without a workspace (scratch in a static device array)."""
    T, k = ids.shape
    off = torch.empty(E + 1, dtype=torch.int32, device=ids.device)
    rs = torch.empty(T * k, dtype=torch.int32, device=ids.device)
    sr = torch.empty(T * k, dtype=torch.int32, device=ids.device)
    _check("moe_permute_noalloc", lib.moe_permute_noalloc(_ptr(ids), T, k, E, _ptr(off), _ptr(rs), _ptr(sr),
                                                          _stream()))
    return off, rs, sr


def grouped_swiglu(x, offsets, row_slot, top_k, gate, up, rows, ws, out=None):
    T, H = x.shape
    h = out if out is not None else torch.empty(rows, gate.out_dim, dtype=torch.bfloat16, device=x.device)
    g, u = gate.struct(), up.struct()
    _check("moe_grouped_w4a16_swiglu",
           lib.moe_grouped_w4a16_swiglu(_ptr(x), T, H, _ptr(offsets), _ptr(row_slot), top_k,
                                        ctypes.byref(g), ctypes.byref(u), 0.0, _ptr(h),
                                        _ptr(ws), ws.numel(), _stream()))
    return h


def grouped_down(h_perm, offsets, row_slot, topk_w, down, ws, out=None):
    rows = h_perm.shape[0]
    y = out if out is not None else torch.empty(rows, down.out_dim, dtype=torch.bfloat16, device=h_perm.device)
    d = down.struct()
    _check("moe_grouped_w4a16_down",
           lib.moe_grouped_w4a16_down(_ptr(h_perm), _ptr(offsets), _ptr(row_slot), _ptr(topk_w), rows,
                                      ctypes.byref(d), _ptr(y), _ptr(ws), ws.numel(), _stream()))
    return y


def unpermute_combine(y_perm, slot_row, T, top_k, shared_out=None, out=None):
    H = y_perm.shape[1]
    y = out if out is not None else torch.empty(T, H, dtype=torch.bfloat16, device=y_perm.device)
    _check("moe_unpermute_combine",
           lib.moe_unpermute_combine(_ptr(y_perm), _ptr(slot_row), T, top_k, H, _ptr(shared_out), _ptr(y),
                                     _stream()))
    return y


def layer_decode(x, layer, ws, out=None):
    T = x.shape[0]
    y = out if out is not None else torch.empty_like(x)
    L = layer.struct()
    _check("moe_layer_decode", lib.moe_layer_decode(_ptr(x), T, ctypes.byref(L), _ptr(y), _ptr(ws),
                                                    ws.numel(), _stream()))
    return y


class LayerGraph:
    """One layer call (moe_layer_forward on these exact tensors) recorded as a CUDA graph;
    launch() replays it on the current stream.  x is read and out written in place at every
    launch; the tensors and the layer's banks are held until the graph is released."""

    def __init__(self, x, layer, ws, out=None):
        self.x, self.layer, self.ws = x, layer, ws
        self.y = out if out is not None else torch.empty_like(x)
        self._L = layer.struct()
        h = _P()
        _check("moe_layer_graph_create", lib.moe_layer_graph_create(
            _ptr(x), x.shape[0], ctypes.byref(self._L), _ptr(self.y), _ptr(ws), ws.numel(), ctypes.byref(h)))
        self._h = h

    def launch(self):
        _check("moe_layer_graph_launch", lib.moe_layer_graph_launch(self._h, _stream()))
        return self.y

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib.moe_layer_graph_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def layer_forward(x, layer, ws, out=None):
    T = x.shape[0]
    y = out if out is not None else torch.empty_like(x)
    L = layer.struct()
    _check("moe_layer_forward", lib.moe_layer_forward(_ptr(x), T, ctypes.byref(L), _ptr(y), _ptr(ws),
                                                      ws.numel(), _stream()))
    return y


def quantize_int4_g128(w):
    rows, cols = w.shape
    packed = torch.empty(rows, cols // 8, dtype=torch.int32, device=w.device)
    scales = torch.empty(rows, cols // 128, dtype=torch.bfloat16, device=w.device)
    _check("moe_quantize_int4_g128",
           lib.moe_quantize_int4_g128(_ptr(w), rows, cols, _ptr(packed), _ptr(scales), _stream()))
    return packed, scales


def quantize_nvfp4(w, ws, global_out=None):
    rows, cols = w.shape
    packed = torch.empty(rows, cols // 2, dtype=torch.uint8, device=w.device)
    scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=w.device)
    g = global_out if global_out is not None else torch.empty(1, dtype=torch.float32, device=w.device)
    _check("moe_quantize_nvfp4",
           lib.moe_quantize_nvfp4(_ptr(w), rows, cols, _ptr(packed), _ptr(scales), _ptr(g), _ptr(ws),
                                  ws.numel(), _stream()))
    return packed, scales, g


def csf_encode(scales):
    """Scale bytes uint8 [E, R, C] (device) -> CSF planes (fixed uint8
    [E, R/16, 16*(1+C/2)], exceptions uint32 [n] as int32 storage, starts int64 [E+1])."""
    E, R, C = scales.shape
    n = int(lib.moe_csf_encode_workspace_bytes(E, R))
    if n == 0:
        raise MoEError("moe_csf_encode_workspace_bytes", -2)
    ws = torch.empty(n, dtype=torch.uint8, device=scales.device)
    _check("moe_workspace_init", lib.moe_workspace_init(_ptr(ws), n, _stream()))
    fixed = torch.empty(E, R // 16, 16 * (1 + C // 2), dtype=torch.uint8, device=scales.device)
    starts = torch.empty(E + 1, dtype=torch.int64, device=scales.device)
    _check("moe_csf_encode", lib.moe_csf_encode(_ptr(scales), E, R, C, _ptr(fixed), _ptr(starts), None, 0,
                                                _ptr(ws), n, _stream()))
    count = int(starts[E].item())
    exc = torch.empty(max(count, 1), dtype=torch.int32, device=scales.device)
    _check("moe_csf_encode", lib.moe_csf_encode(_ptr(scales), E, R, C, _ptr(fixed), _ptr(starts), _ptr(exc), count,
                                                _ptr(ws), n, _stream()))
    st = read_status(ws)
    if st != 0:
        raise MoEError("moe_csf_encode (device)", st)
    return fixed, exc[:count], starts


def csf_decode(fixed, exceptions, starts, R, C, expert_offsets=None, out=None):
    E = fixed.shape[0]
    sc = out if out is not None else torch.empty(E, R, C, dtype=torch.uint8, device=fixed.device)
    exc = exceptions if exceptions.numel() else torch.zeros(1, dtype=torch.int32, device=fixed.device)
    _check("moe_csf_decode", lib.moe_csf_decode(_ptr(fixed), _ptr(exc), _ptr(starts), E, R, C, _ptr(expert_offsets),
                                                _ptr(sc), _stream()))
    return sc


def quantize_nvfp4_act(x, g):
    """Activations bf16 [rows, cols] with per-row globals g fp32 [rows] (device) ->
    (packed uint8 [rows, cols/2], scales uint8 [rows, cols/16])."""
    rows, cols = x.shape
    packed = torch.empty(rows, cols // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=x.device)
    _check("moe_quantize_nvfp4_act",
           lib.moe_quantize_nvfp4_act(_ptr(x), rows, cols, _ptr(g), _ptr(packed), _ptr(scales), _stream()))
    return packed, scales
