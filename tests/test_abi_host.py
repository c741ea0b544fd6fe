"""C ABI checks that need no GPU: the library loads, exports every function
the public header declares, and rejects bad arguments on the host before
touching the device (fail closed); with no device present, valid calls fail
with MOE_ERR_CUDA rather than running anything on the CPU."""
import ctypes
import os
import re

import pytest

import fp8_blockwise_routed_b200 as fm

V = ctypes.c_void_p
A = V(0x10000)          # 16-byte aligned stand-in address (never dereferenced)
MIS = V(0x10001)        # misaligned


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(fm.LIB_PATH):
        from fp8_blockwise_routed_b200 import build
        build.build()
    return fm.lib()


def test_exports_every_declared_symbol(L):
    names = fm.declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n


def test_header_declares_the_four_path_calls():
    src = open(fm.HEADER_PATH).read()
    for n in ("moe_route", "moe_quant_act", "moe_grouped_ffn", "moe_combine"):
        assert re.search(rf"MOE_API int {n}\(", src), n


def test_status_strings(L):
    for code, name in fm.STATUS.items():
        assert L.moe_status_string(code).decode() == name
    assert L.moe_abi_version() >> 16 == 1


def test_route_validation(L):
    ws = 1 << 20
    assert L.moe_route(A, 4, 0, 1, A, A, A, A, A, ws, None) == 1        # E = 0
    assert L.moe_route(A, 4, 2000, 1, A, A, A, A, A, ws, None) == 1     # E > 1024
    assert L.moe_route(A, 4, 8, 9, A, A, A, A, A, ws, None) == 1        # top_k > E
    assert L.moe_route(A, 4, 64, 33, A, A, A, A, A, ws, None) == 1      # top_k > 32
    assert L.moe_route(A, -1, 8, 2, A, A, A, A, A, ws, None) == 1       # T < 0
    assert L.moe_route(MIS, 4, 8, 2, A, A, A, A, A, ws, None) == 3      # misaligned
    need = L.moe_route_workspace_bytes(4, 8, 2)
    assert L.moe_route(A, 4, 8, 2, A, A, A, A, A, need - 1, None) == 4  # workspace
    assert L.moe_route(A, 4, 8, 2, A, A, A, A, A, need, None) == 5      # no device here


def test_quant_validation(L):
    assert L.moe_quant_act(A, 4, 100, A, A, None) == 1
    assert L.moe_quant_act(A, 4, 0, A, A, None) == 1
    assert L.moe_quant_act(A, 4, 128 * 200, A, A, None) == 1
    assert L.moe_quant_act(MIS, 4, 128, A, A, None) == 3
    assert L.moe_quant_act(A, 0, 128, A, A, None) == 0               # T = 0: no-op
    assert L.moe_quant_act(A, 4, 128, A, A, None) == 5               # no device here


def _ffn(L, T=4, H=256, k=2, E=8, I=128, ws=None, ptr=A):
    if ws is None:
        ws = L.moe_ffn_workspace_bytes(T, H, I, E, k)
    return L.moe_grouped_ffn(ptr, A, T, H, A, A, k, A, A, E, I, A, A, A, A, A, A, A, A, ws, None, None)


def test_ffn_validation(L):
    assert _ffn(L, H=200) == 1
    assert _ffn(L, I=0) == 1
    assert _ffn(L, I=100) == 2          # I % 16 != 0: unsupported (TMA strides)
    assert _ffn(L, I=16384) == 1
    assert _ffn(L, k=0) == 1
    assert _ffn(L, k=9, E=8) == 1
    assert _ffn(L, ptr=MIS) == 3
    assert _ffn(L, ws=64) == 4
    assert _ffn(L) == 5                 # no device here


def test_quant_mx_validation(L):
    assert L.moe_quant_act_mx(A, 4, 100, A, A, None) == 1           # H % 32 != 0
    assert L.moe_quant_act_mx(A, 4, 16, A, A, None) == 1            # H < 32
    assert L.moe_quant_act_mx(A, -1, 64, A, A, None) == 1
    assert L.moe_quant_act_mx(A, 4, 64, MIS, A, None) == 3
    assert L.moe_quant_act_mx(A, 0, 64, A, A, None) == 0             # T = 0: no-op
    assert L.moe_quant_act_mx(A, 4, 64, A, A, None) == 5             # no device here


def _ffn_mx(L, T=4, H=256, k=2, E=8, I=128, ws=None, ptr=A):
    if ws is None:
        ws = L.moe_ffn_mx_workspace_bytes(T, H, I, E, k)
    return L.moe_grouped_ffn_mx(ptr, A, T, H, A, A, k, A, A, E, I, A, A, A, A, A, A, A, A, ws, None, None)


def test_ffn_mx_validation(L):
    assert _ffn_mx(L, H=200) == 1       # H % 128 != 0
    assert _ffn_mx(L, I=96) == 1        # I < 128
    assert _ffn_mx(L, I=144) == 2       # I % 32 != 0: unsupported (one scale per 32 columns)
    assert _ffn_mx(L, I=16384) == 1
    assert _ffn_mx(L, k=0) == 1
    assert _ffn_mx(L, k=9, E=8) == 1
    assert _ffn_mx(L, ptr=MIS) == 3
    assert _ffn_mx(L, ws=64) == 4
    assert _ffn_mx(L) == 5              # no device here
    ws = L.moe_combine_workspace_bytes()
    assert L.moe_debug_grouped_down_mx(A, A, 4, 256, 2, A, A, A, 8, 144, A, A, A, A, ws, None) == 2
    assert L.moe_debug_grouped_down_mx(A, A, 4, 256, 2, A, A, A, 8, 128, A, A, A, A, 8, None) == 4


def test_pack_scales_validation(L):
    assert L.moe_mx_packed_scales_bytes(3, 70, 5120) == 3 * 10 * 70 * 16
    assert L.moe_mx_packed_scales_bytes(2, 33, 192) == 2 * 1 * 33 * 16
    assert L.moe_mx_packed_scales_bytes(1, 5, 100) == 0             # K % 32 != 0
    assert L.moe_mx_pack_scales(A, 2, 33, 100, A, None) == 1
    assert L.moe_mx_pack_scales(A, 2, 0, 192, A, None) == 1
    assert L.moe_mx_pack_scales(A, 2, 33, 192, MIS, None) == 3
    assert L.moe_mx_pack_scales(A, 0, 33, 192, A, None) == 0         # E = 0: no-op
    assert L.moe_mx_pack_scales(A, 2, 33, 192, A, None) == 5         # no device here


def test_mx_workspace_layout(L):
    """The MX FFN workspace holds the expert-ordered codes, the intermediate
    and both K-group-major scale arrays; the intermediate accessor points
    inside it, at offsets that grow with T."""
    T, H, I, E, k = 4096, 5120, 1536, 256, 8
    P = T * k
    b = L.moe_ffn_mx_workspace_bytes(T, H, I, E, k)
    Ip = 1536
    assert b >= P * (H + Ip) + P * 16 * ((H + 511) // 512 + (Ip + 511) // 512)
    hc, hs = V(), V()
    assert L.moe_ffn_mx_intermediate(A, T, H, I, k, ctypes.byref(hc), ctypes.byref(hs)) == 0
    assert A.value < hc.value < hs.value < A.value + b
    assert hs.value - hc.value >= P * Ip


def test_combine_validation(L):
    ws = L.moe_combine_workspace_bytes()
    f = ctypes.c_float(1.0)
    assert L.moe_combine(A, A, 4, 100, 2, 8, f, A, None, A, ws, None) == 1
    assert L.moe_combine(A, A, 4, 256, 2, 8, f, A, None, A, 8, None) == 4
    assert L.moe_combine(A, A, 4, 256, 2, 8, f, MIS, None, A, ws, None) == 3
    assert L.moe_combine(A, A, 4, 256, 2, 8, f, A, None, A, ws, None) == 5


def test_workspace_sizes_grow_with_T(L):
    a = L.moe_ffn_workspace_bytes(64, 256, 128, 8, 2)
    b = L.moe_ffn_workspace_bytes(4096, 5120, 1536, 256, 8)
    assert 0 < a < b
    # gathered A rows + intermediate codes dominate: about P*(H + Ip) bytes
    P = 4096 * 8
    assert b >= P * (5120 + 1536)
    assert L.moe_route_workspace_bytes(16384, 256, 8) > L.moe_route_workspace_bytes(64, 8, 2)


def test_binding_has_no_fallback():
    """The binding module imports nothing from the oracle and exposes no
    CPU implementation of the path."""
    src = open(fm.__file__).read()
    assert "import oracle" not in src and "from oracle" not in src
    for f in os.listdir(os.path.join(os.path.dirname(fm.__file__), "csrc")):
        text = open(os.path.join(os.path.dirname(fm.__file__), "csrc", f)).read()
        assert "oracle" not in text.lower(), f
