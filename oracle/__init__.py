"""CPU oracle for the 4-bit routed-expert MoE layer of Step-5-Preview.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  It shares no
code with the CUDA path.  The arithmetic lives in ``moe_oracle.c`` (each
function cites the page passage it follows); this module only marshals numpy
arrays through ctypes.

bf16 tensors are passed as their uint16 bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        F = ctypes.c_float
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = F
        L.oracle_f32_to_bf16.argtypes = [F]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f32.restype = F
        L.oracle_set_x_f16.argtypes = [I]
        L.oracle_set_x_f16.restype = None
        L.oracle_set_threads.argtypes = [I]
        L.oracle_set_threads.restype = I
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = F
        L.oracle_e2m1_encode.argtypes = [F]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = F
        L.oracle_e4m3_encode_nonneg.argtypes = [F]
        L.oracle_e4m3_encode_nonneg.restype = ctypes.c_uint8
        L.oracle_quant_int4_g128.argtypes = [P, I64, I64, P, P, P, P, I]
        L.oracle_quant_int4_g128.restype = None
        L.oracle_dequant_int4_g128.argtypes = [P, P, I64, I64, P]
        L.oracle_dequant_int4_g128.restype = None
        L.oracle_quant_nvfp4.argtypes = [P, I64, I64, P, P, P]
        L.oracle_quant_nvfp4.restype = None
        L.oracle_dequant_nvfp4.argtypes = [P, P, F, I64, I64, P]
        L.oracle_dequant_nvfp4.restype = None
        L.oracle_dequant_expert.argtypes = [P, I, P]
        L.oracle_dequant_expert.restype = None
        L.oracle_route.argtypes = [P, I64, I64, P, P, I64, I, P, P, P]
        L.oracle_route.restype = None
        L.oracle_permute.argtypes = [P, I64, I, I64, P, P, P]
        L.oracle_permute.restype = I
        L.oracle_moe_forward.argtypes = [P, I64, I64, I64, I, P, P, P, P, P, P, P, P, P, I64, P]
        L.oracle_moe_forward.restype = I
        L.oracle_grouped_swiglu.argtypes = [P, I64, I64, I, P, P, P, P, P, I64, P]
        L.oracle_grouped_swiglu.restype = None
        L.oracle_grouped_down.argtypes = [P, I64, I64, P, P, P, P, P, I64, P]
        L.oracle_grouped_down.restype = None
        L.oracle_combine.argtypes = [P, P, I64, I, I64, P, P]
        L.oracle_combine.restype = None
        L.oracle_act_quant_nvfp4.argtypes = [P, I64, I64, P, P, P, P]
        L.oracle_act_quant_nvfp4.restype = None
        L.oracle_grouped_swiglu_w4a4.argtypes = [P, I64, I64, I, P, P, P, P, P, P, I64, P]
        L.oracle_grouped_swiglu_w4a4.restype = None
        L.oracle_grouped_down_w4a4.argtypes = [P, I64, I64, P, P, P, P, P, P, I64, P]
        L.oracle_grouped_down_w4a4.restype = None
        L.oracle_moe_forward_w4a4.argtypes = [P, I64, I64, I64, I, P, P, P, P, P, P, P, P, P, P, P, I64, P]
        L.oracle_moe_forward_w4a4.restype = I
        L.oracle_csf_encode.argtypes = [P, I64, I64, I64, P, P, P]
        L.oracle_csf_encode.restype = I64
        L.oracle_csf_decode.argtypes = [P, P, P, I64, I64, I64, P]
        L.oracle_csf_decode.restype = None
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


FMT_INT4, FMT_NVFP4, FMT_BF16 = 0, 1, 2


class _Bank(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("out", ctypes.c_int32),
                ("in_", ctypes.c_int32), ("packed", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_void_p)]


class Bank:
    """An expert bank in the pages' fused layout [E, out, in].

    int4:  packed int32 [E,out,in/8], scales uint16(bf16) [E,out,in/128]
    nvfp4: packed uint8 [E,out,in/2], scales uint8(E4M3) [E,out,in/16], global fp32 [E]
    bf16:  packed uint16 [E,out,in]
    """

    def __init__(self, fmt, packed, scales=None, global_scale=None, out=None, in_=None):
        self.fmt = fmt
        self.packed = packed
        self.scales = scales
        self.global_scale = global_scale
        E = packed.shape[0]
        if out is None:
            out = packed.shape[1]
        if in_ is None:
            in_ = packed.shape[2] * {FMT_INT4: 8, FMT_NVFP4: 2, FMT_BF16: 1}[fmt]
        self.E, self.out, self.in_ = E, out, in_

    def _struct(self):
        s = _Bank(self.fmt, self.E, self.out, self.in_, _p(self.packed),
                  _p(self.scales), _p(self.global_scale))
        return s


def bf16_to_f32(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f16_to_f32(bits):
    return lib().oracle_f16_to_f32(int(bits))


class x_f16:
    """Context: the layer's input activations x are fp16 bits instead of bf16
    (route, moe_forward, grouped_swiglu and the W4A4 gate/up read x that way)."""

    def __enter__(self):
        lib().oracle_set_x_f16(1)
        return self

    def __exit__(self, *a):
        lib().oracle_set_x_f16(0)


def set_threads(n):
    """OpenMP threads of later oracle calls (n <= 0: one per host core); returns the count in effect.
    For timing only: results do not depend on it."""
    return int(lib().oracle_set_threads(int(n)))


def f32_to_bf16_scalar(v):
    return lib().oracle_f32_to_bf16(float(v))


def e2m1_decode(code):
    return lib().oracle_e2m1_decode(int(code))


def e2m1_encode(v):
    return lib().oracle_e2m1_encode(float(v))


def e4m3_decode(b):
    return lib().oracle_e4m3_decode(int(b))


def e4m3_encode(v):
    return lib().oracle_e4m3_encode_nonneg(float(v))


def quant_int4_g128(w_bits, want_q=False, want_ratio=False, max_abs_only=False):
    """bf16 bits [rows, cols] -> (packed int32 [rows, cols/8], scales uint16 [rows, cols/128]
    [, q int8 [rows, cols]] [, ratio index int32 [rows, cols/128]]).

    max_abs_only: use the single ratio 1.00 (the page's max-abs baseline row)
    instead of the 17-ratio clip search."""
    w = _c(w_bits, np.uint16)
    rows, cols = w.shape
    assert cols % 128 == 0
    packed = np.empty((rows, cols // 8), np.int32)
    scales = np.empty((rows, cols // 128), np.uint16)
    q = np.empty((rows, cols), np.int8) if want_q else None
    ri = np.empty((rows, cols // 128), np.int32) if want_ratio else None
    lib().oracle_quant_int4_g128(_p(w), rows, cols, _p(packed), _p(scales), _p(q), _p(ri),
                                 16 if max_abs_only else 0)
    out = [packed, scales]
    if want_q:
        out.append(q)
    if want_ratio:
        out.append(ri)
    return tuple(out)


def dequant_int4_g128(packed, scales):
    packed = _c(packed, np.int32)
    scales = _c(scales, np.uint16)
    rows = packed.shape[0]
    cols = packed.shape[1] * 8
    out = np.empty((rows, cols), np.float32)
    lib().oracle_dequant_int4_g128(_p(packed), _p(scales), rows, cols, _p(out))
    return out


def quant_nvfp4(w_bits):
    """bf16 bits [rows, cols] (one expert matrix) -> (packed uint8 [rows, cols/2],
    scales uint8 [rows, cols/16], global float)."""
    w = _c(w_bits, np.uint16)
    rows, cols = w.shape
    assert cols % 16 == 0
    packed = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    g = np.zeros(1, np.float32)
    lib().oracle_quant_nvfp4(_p(w), rows, cols, _p(packed), _p(scales), _p(g))
    return packed, scales, float(g[0])


def dequant_nvfp4(packed, scales, global_scale):
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint8)
    rows = packed.shape[0]
    cols = packed.shape[1] * 2
    out = np.empty((rows, cols), np.float32)
    lib().oracle_dequant_nvfp4(_p(packed), _p(scales), float(global_scale), rows, cols, _p(out))
    return out


def dequant_expert(bank, e):
    out = np.empty((bank.out, bank.in_), np.float32)
    s = bank._struct()
    lib().oracle_dequant_expert(ctypes.addressof(s), int(e), _p(out))
    return out


def route(x_bits, router_w, bias, k, want_scores=False):
    """x bf16 bits [T,H], router_w fp32 [E,H], bias fp32 [E] or None ->
    (ids int32 [T,k], w fp32 [T,k] [, scores fp32 [T,E]])."""
    x = _c(x_bits, np.uint16)
    Wr = _c(router_w, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    sc = np.empty((T, E), np.float32) if want_scores else None
    lib().oracle_route(_p(x), T, H, _p(Wr), _p(b), E, k, _p(ids), _p(w), _p(sc))
    return (ids, w, sc) if want_scores else (ids, w)


def permute(ids, E):
    """ids int32 [T,k] -> (offsets int32 [E+1], row_slot int32 [T*k], slot_row int32 [T*k])."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    offsets = np.empty(E + 1, np.int32)
    rs = np.empty(T * k, np.int32)
    sr = np.empty(T * k, np.int32)
    rc = lib().oracle_permute(_p(ids), T, k, E, _p(offsets), _p(rs), _p(sr))
    if rc != 0:
        raise ValueError("expert id out of range")
    return offsets, rs, sr


def moe_forward(x_bits, ids, topk_w, gate, up, down, shared=None, tokens=None):
    """fp64 layer output for the listed tokens (default: all) -> float64 [n, H].

    shared: None or a (gate, up, down) tuple of BF16 banks with E=1."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    ids = _c(ids, np.int32)
    w = _c(topk_w, np.float32)
    k = ids.shape[1]
    F = gate.out
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tok = _c(tokens, np.int32)
    n = tok.shape[0]
    y = np.empty((n, H), np.float64)
    sg, su, sd = (shared if shared is not None else (None, None, None))
    structs = [b._struct() if b is not None else None for b in (gate, up, down, sg, su, sd)]
    refs = [ctypes.addressof(s) if s is not None else None for s in structs]
    rc = lib().oracle_moe_forward(_p(x), T, H, F, k, _p(ids), _p(w), *refs, _p(tok), n, _p(y))
    if rc != 0:
        raise ValueError("expert id out of range")
    return y


def grouped_swiglu(x_bits, offsets, row_slot, k, gate, up, rows):
    """h[i, :] for permuted rows `rows` (fp64 [n, F])."""
    x = _c(x_bits, np.uint16)
    H = x.shape[1]
    F = gate.out
    rows = _c(rows, np.int32)
    h = np.empty((rows.shape[0], F), np.float64)
    g, u = gate._struct(), up._struct()
    lib().oracle_grouped_swiglu(_p(x), H, F, k, _p(_c(offsets, np.int32)), _p(_c(row_slot, np.int32)),
                                ctypes.addressof(g), ctypes.addressof(u), _p(rows), rows.shape[0], _p(h))
    return h


def grouped_down(h_bits, offsets, row_slot, topk_w, down, rows):
    """y[i, :] for permuted rows `rows` (fp64 [n, H]); topk_w indexed by slot or None."""
    hb = _c(h_bits, np.uint16)
    F = hb.shape[1]
    H = down.out
    rows = _c(rows, np.int32)
    y = np.empty((rows.shape[0], H), np.float64)
    d = down._struct()
    tw = None if topk_w is None else _c(topk_w, np.float32)
    lib().oracle_grouped_down(_p(hb), F, H, _p(_c(offsets, np.int32)), _p(_c(row_slot, np.int32)), _p(tw),
                              ctypes.addressof(d), _p(rows), rows.shape[0], _p(y))
    return y


def combine(y_perm_bits, slot_row, T, k, shared_bits=None):
    yp = _c(y_perm_bits, np.uint16)
    H = yp.shape[1]
    y = np.empty((T, H), np.float64)
    sh = None if shared_bits is None else _c(shared_bits, np.uint16)
    lib().oracle_combine(_p(yp), _p(_c(slot_row, np.int32)), T, k, H, _p(sh), _p(y))
    return y


def csf_encode(scales):
    """E4M3 scale bytes uint8 [E, R, C] -> (fixed uint8 [E, R/16, 16*(1+C/2)],
    exceptions uint32 [n], starts int64 [E+1]) in the compressed scale format."""
    sc = _c(scales, np.uint8)
    E, R, C = sc.shape
    assert R % 16 == 0 and C % 2 == 0
    fixed = np.empty((E, R // 16, 16 * (1 + C // 2)), np.uint8)
    starts = np.empty(E + 1, np.int64)
    n = lib().oracle_csf_encode(_p(sc), E, R, C, _p(fixed), _p(starts), None)
    exc = np.empty(n, np.uint32)
    lib().oracle_csf_encode(_p(sc), E, R, C, _p(fixed), _p(starts), _p(exc))
    return fixed, exc, starts


def csf_decode(fixed, exceptions, starts, R, C):
    fixed = _c(fixed, np.uint8)
    E = fixed.shape[0]
    out = np.empty((E, R, C), np.uint8)
    lib().oracle_csf_decode(_p(fixed), _p(_c(exceptions, np.uint32)), _p(_c(starts, np.int64)), E, R, C, _p(out))
    return out


def act_quant_nvfp4(x_bits, g):
    """bf16 bits [rows, cols], global fp32 per row (scalar or [rows]) ->
    (packed uint8 [rows, cols/2], scales uint8 [rows, cols/16], dequantised fp32 [rows, cols])."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    gg = _c(np.broadcast_to(np.asarray(g, np.float32), (rows,)), np.float32)
    packed = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    xq = np.empty((rows, cols), np.float32)
    lib().oracle_act_quant_nvfp4(_p(x), rows, cols, _p(gg), _p(packed), _p(scales), _p(xq))
    return packed, scales, xq


def grouped_swiglu_w4a4(x_bits, offsets, row_slot, k, gate, up, in_scale, rows):
    x = _c(x_bits, np.uint16)
    H = x.shape[1]
    F = gate.out
    rows = _c(rows, np.int32)
    h = np.empty((rows.shape[0], F), np.float64)
    g, u = gate._struct(), up._struct()
    lib().oracle_grouped_swiglu_w4a4(_p(x), H, F, k, _p(_c(offsets, np.int32)), _p(_c(row_slot, np.int32)),
                                     ctypes.addressof(g), ctypes.addressof(u), _p(_c(in_scale, np.float32)),
                                     _p(rows), rows.shape[0], _p(h))
    return h


def grouped_down_w4a4(h_bits, offsets, row_slot, topk_w, down, in_scale, rows):
    hb = _c(h_bits, np.uint16)
    F = hb.shape[1]
    H = down.out
    rows = _c(rows, np.int32)
    y = np.empty((rows.shape[0], H), np.float64)
    d = down._struct()
    tw = None if topk_w is None else _c(topk_w, np.float32)
    lib().oracle_grouped_down_w4a4(_p(hb), F, H, _p(_c(offsets, np.int32)), _p(_c(row_slot, np.int32)), _p(tw),
                                   ctypes.addressof(d), _p(_c(in_scale, np.float32)), _p(rows), rows.shape[0], _p(y))
    return y


def moe_forward_w4a4(x_bits, ids, topk_w, gate, up, down, in_gu, in_dn, shared=None, tokens=None):
    """fp64 W4A4 layer output for the listed tokens (default: all) -> float64 [n, H]."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    ids = _c(ids, np.int32)
    w = _c(topk_w, np.float32)
    k = ids.shape[1]
    F = gate.out
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tok = _c(tokens, np.int32)
    n = tok.shape[0]
    y = np.empty((n, H), np.float64)
    sg, su, sd = (shared if shared is not None else (None, None, None))
    structs = [b._struct() if b is not None else None for b in (gate, up, down, sg, su, sd)]
    refs = [ctypes.addressof(s) if s is not None else None for s in structs]
    rc = lib().oracle_moe_forward_w4a4(_p(x), T, H, F, k, _p(ids), _p(w), refs[0], refs[1], refs[2],
                                       _p(_c(in_gu, np.float32)), _p(_c(in_dn, np.float32)), refs[3], refs[4],
                                       refs[5], _p(tok), n, _p(y))
    if rc != 0:
        raise ValueError("expert id out of range")
    return y
