"""The C-ABI library loads, exports every function the public header declares,
and rejects bad arguments on the host before launching anything (no GPU
needed: every call below returns during argument validation)."""
import ctypes

from weight_only_bit_route_b200 import moe

P = ctypes.c_void_p
FAKE = P(0x10000)          # aligned, never dereferenced by the host checks
MIS = P(0x10008)           # 8-byte aligned only


def test_exports_every_declared_function():
    names = moe.declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(moe.lib, n), n
    for must in ("moe_route_topk", "moe_permute", "moe_grouped_w4a16_swiglu", "moe_grouped_w4a16_down",
                 "moe_unpermute_combine", "moe_layer_decode"):
        assert must in names


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert moe.lib.moe_status_string(code)
    assert moe.lib.moe_status_string(12345) == b"unknown status"


def test_workspace_bytes():
    assert moe.workspace_bytes(8, 4096, 352, 1536, 8) > 0
    assert moe.workspace_bytes(8, 4096, 352, 1536, 9) == 0      # top_k > 8
    assert moe.workspace_bytes(8, 4000, 352, 1536, 8) == 0      # H % 128
    assert moe.workspace_bytes(8, 4096, 2000, 1536, 8) == 0     # E > 1024
    assert moe.workspace_bytes(-1, 4096, 352, 1536, 8) == 0
    big = moe.workspace_bytes(8192, 4096, 352, 1536, 8)
    # holds at least the permuted down output (T*k rows of H bf16)
    assert big >= 8192 * 8 * 4096 * 2


def test_route_topk_argument_errors():
    L = moe.lib
    assert L.moe_route_topk(FAKE, 0, 4096, FAKE, None, 352, 8, FAKE, FAKE, FAKE, 1 << 20, None) == 0
    assert L.moe_route_topk(None, 4, 4096, FAKE, None, 352, 8, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.moe_route_topk(MIS, 4, 4096, FAKE, None, 352, 8, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.moe_route_topk(FAKE, 4, 4096, FAKE, None, 352, 9, FAKE, FAKE, FAKE, 1 << 20, None) == -2
    assert L.moe_route_topk(FAKE, 4, 4000, FAKE, None, 352, 8, FAKE, FAKE, FAKE, 1 << 20, None) == -2
    assert L.moe_route_topk(FAKE, 4, 4096, FAKE, None, 352, 8, FAKE, FAKE, FAKE, 16, None) == -5
    assert L.moe_route_topk(FAKE, 4, 4096, FAKE, None, 352, 8, FAKE, FAKE, None, 1 << 20, None) == -5


def _bank(fmt, E, out, inn, packed=FAKE, scales=FAKE, glob=FAKE):
    return moe.QWeight(fmt, E, out, inn, packed, scales, glob)


def _layer(**kw):
    E, H, F = 352, 4096, 1536
    d = dict(gate=_bank(0, E, F, H), up=_bank(0, E, F, H), down=_bank(0, E, H, F),
             sh_gate=_bank(2, 1, F, H), sh_up=_bank(2, 1, F, H), sh_down=_bank(2, 1, H, F),
             router_w=FAKE, router_bias=None, E=E, H=H, F=F, top_k=8, swiglu_limit=0.0)
    d.update(kw)
    return moe.Layer(**d)


def test_layer_argument_errors():
    L = moe.lib
    call = lambda lay, T=8, ws=FAKE, wsb=1 << 34: L.moe_layer_decode(FAKE, T, ctypes.byref(lay), FAKE, ws, wsb, None)
    assert call(_layer(), T=0) == 0
    assert call(_layer(swiglu_limit=7.0)) == -2
    assert call(_layer(top_k=9)) == -2
    assert call(_layer(F=1500)) == -2
    assert call(_layer(gate=_bank(0, 352, 1536, 4096, packed=MIS))) == -1
    assert call(_layer(gate=_bank(1, 352, 1536, 4096, glob=None), up=_bank(1, 352, 1536, 4096),
                       down=_bank(1, 352, 4096, 1536))) == -1
    assert call(_layer(gate=_bank(0, 352, 1536, 4096, scales=None))) == -1
    assert call(_layer(down=_bank(1, 352, 4096, 1536))) == -2          # mixed formats
    assert call(_layer(sh_gate=_bank(0, 1, 1536, 4096))) == -2          # shared must be bf16
    assert call(_layer(gate=_bank(0, 351, 1536, 4096))) == -1           # E mismatch
    assert call(_layer(), ws=None) == -5
    assert call(_layer(), wsb=1024) == -5
    assert call(_layer(), T=65) == -2                                   # decode entry limit
    assert L.moe_layer_decode(None, 8, ctypes.byref(_layer()), FAKE, FAKE, 1 << 34, None) == -1


def test_layer_graph_argument_errors():
    """The recorded layer's calls refuse bad arguments before any CUDA call, and leave the handle empty."""
    L = moe.lib
    h = P(0x1234)

    def create(lay, T=8, ws=FAKE, wsb=1 << 34, out=True):
        h.value = 0x1234
        return L.moe_layer_graph_create(FAKE, T, ctypes.byref(lay), FAKE, ws, wsb, ctypes.byref(h) if out else None)

    assert create(_layer(), out=False) == -1
    assert create(_layer(), T=0) == -1 and not h.value                 # nothing to record
    assert create(_layer(swiglu_limit=7.0)) == -2 and not h.value
    assert create(_layer(gate=_bank(0, 351, 1536, 4096))) == -1 and not h.value
    assert create(_layer(), ws=None) == -5 and not h.value
    assert L.moe_layer_graph_launch(None, None) == -1
    assert L.moe_layer_graph_destroy(None) == 0


def test_step_argument_errors():
    L = moe.lib
    g = _bank(0, 352, 1536, 4096)
    assert L.moe_grouped_w4a16_swiglu(FAKE, 8, 4096, FAKE, FAKE, 8, ctypes.byref(g), ctypes.byref(g), 1.0,
                                      FAKE, FAKE, 1 << 30, None) == -2
    assert L.moe_grouped_w4a16_swiglu(FAKE, 8, 4096, None, FAKE, 8, ctypes.byref(g), ctypes.byref(g), 0.0,
                                      FAKE, FAKE, 1 << 30, None) == -1
    d = _bank(0, 352, 4096, 1536)
    assert L.moe_grouped_w4a16_down(FAKE, FAKE, FAKE, None, 0, ctypes.byref(d), FAKE, FAKE, 1 << 30, None) == 0
    assert L.moe_grouped_w4a16_down(MIS, FAKE, FAKE, None, 64, ctypes.byref(d), FAKE, FAKE, 1 << 30, None) == -1
    assert L.moe_unpermute_combine(FAKE, FAKE, 4, 8, 4000, None, FAKE, None) == -2
    assert L.moe_unpermute_combine(FAKE, None, 4, 8, 4096, None, FAKE, None) == -1
    assert L.moe_permute(FAKE, 4, 9, 352, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -2
    assert L.moe_permute(FAKE, 4, 8, 352, None, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.moe_quantize_int4_g128(FAKE, 4, 100, FAKE, FAKE, None) == -2
    assert L.moe_quantize_nvfp4(FAKE, 4, 32, FAKE, FAKE, FAKE, None, 0, None) == -5
