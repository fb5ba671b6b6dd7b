"""The C-ABI library builds, loads and exports every declared symbol; host-side
validation returns error codes (no GPU needed: none of these calls launches)."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_30_b200 import binding as B
from mixture_experts_layer_30_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.lib()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            src = open(os.path.join(inc, fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(B.SIGNATURES), set(names) - set(B.SIGNATURES)


def test_workspace_bytes_and_validation(lib):
    s = B.make_shape(8192, 6144, 512, 256, 12, 2048, "bf16")
    n = B.workspace_bytes(s)
    # logits + h dominate: T*E*4 + T*K*I*2
    assert n >= 8192 * 768 * 4 + 8192 * 12 * 2048 * 2
    for bad in (B.make_shape(8, 64, 0, 2, 1, 8, "f32"),      # N < 1
                B.make_shape(8, 64, 4, 2, 7, 8, "f32"),      # K > N+Z
                B.make_shape(8, 64, 4, 2, 0, 8, "f32"),      # K < 1
                B.make_shape(8, 62, 4, 2, 2, 8, "f32"),      # rows not 16-byte multiples
                B.make_shape(8, 64, 1000, 100, 2, 8, "f32"),  # E > 1024
                B.make_shape(-1, 64, 4, 2, 2, 8, "f32")):
        assert lib.moe_workspace_bytes(ctypes.byref(bad)) == 0


def test_tiled_layout_validation(lib):
    ok = B.make_shape(16, 256, 4, 2, 2, 128, "bf16", B.WEIGHTS_TILED)
    assert lib.moe_workspace_bytes(ctypes.byref(ok)) > 0
    for bad in (B.make_shape(16, 256, 4, 2, 2, 128, "f32", B.WEIGHTS_TILED),   # bf16 only
                B.make_shape(16, 192, 4, 2, 2, 128, "bf16", B.WEIGHTS_TILED),  # d % 128
                B.make_shape(16, 256, 4, 2, 2, 64, "bf16", B.WEIGHTS_TILED),   # I % 128
                B.make_shape(16, 256, 4, 2, 2, 128, "bf16", 5)):               # unknown
        assert lib.moe_workspace_bytes(ctypes.byref(bad)) == 0
    fake = ctypes.c_void_p(0x10000)
    assert lib.moe_pack_weights(2, 100, 64, B.MOE_BF16, fake, fake, None) == 1   # rows % 128
    assert lib.moe_pack_weights(2, 128, 96, B.MOE_BF16, fake, fake, None) == 1   # cols % 64
    assert lib.moe_pack_weights(2, 128, 64, B.MOE_F32, fake, fake, None) == 2    # bf16 only
    assert lib.moe_pack_weights(2, 128, 64, B.MOE_BF16, fake, ctypes.c_void_p(0x10000 + 4096),
                                None) == 1                                      # overlap
    assert b"overlap" in lib.moe_last_error()


def test_invalid_arguments_return_codes(lib):
    s = B.make_shape(16, 64, 4, 2, 2, 32, "f32")
    nb = B.workspace_bytes(s)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    # NULL shape
    assert lib.moe_route(None, fake, fake, fake, None, fake, fake, fake, fake, None, None, fake,
                         nb, None) == 1
    # NULL workspace
    assert lib.moe_route(ctypes.byref(s), fake, fake, fake, None, fake, fake, fake, fake, None,
                         None, None, nb, None) == 1
    assert b"workspace" in lib.moe_last_error()
    # workspace too small
    assert lib.moe_permute(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake,
                           nb - 256, None) == 3
    # misaligned workspace
    assert lib.moe_expert_ffn(ctypes.byref(s), fake, fake, fake, fake, fake, fake,
                              ctypes.c_void_p(0x10008), nb, None) == 1
    # NULL operand
    assert lib.moe_expert_gate_up(ctypes.byref(s), None, fake, fake, fake, fake, fake, nb,
                                  None) == 1
    assert b"x_perm" in lib.moe_last_error()
    # route + dispatch layout: the layout outputs are required
    assert lib.moe_route_dispatch(ctypes.byref(s), fake, fake, fake, None, fake, fake, fake,
                                  fake, None, None, None, fake, fake, fake, nb, None) == 1
    assert b"offsets" in lib.moe_last_error()
    assert lib.moe_route_dispatch(ctypes.byref(s), fake, fake, fake, None, fake, fake, fake,
                                  fake, None, None, fake, None, fake, fake, nb, None) == 1
    assert b"row_token" in lib.moe_last_error()
    # bias update argument checks
    assert lib.moe_bias_update(0, 2, fake, 16, 2, 1.0, 0.1, fake, None) == 1
    assert lib.moe_bias_update(4, 2, fake, 0, 2, 1.0, 0.1, fake, None) == 1
    assert lib.moe_bias_update(4, 2, fake, 16, 9, 1.0, 0.1, fake, None) == 1
    # bad dtype code
    bad = B.Shape(16, 64, 4, 2, 2, 32, 7)
    assert lib.moe_combine(ctypes.byref(bad), fake, fake, fake, fake, fake, 1.0, fake, None) == 1


def test_lb_stats_validation(lib):
    fake = ctypes.c_void_p(0x10000)
    args = dict(N=8, Z=4, D=2, T=16, K=3, K_e=2.0)

    def call(**over):
        a = dict(args, **over)
        return lib.moe_lb_stats(a["N"], a["Z"], a["D"], fake, fake, a["T"], a["K"], a["K_e"],
                                0.01, fake, fake, None, None)
    assert call(D=3) == 1        # D must divide N
    assert call(Z=0) == 1        # the zero-expert group must exist
    assert call(K_e=3.0) == 1    # K_e < K
    assert call(K_e=0.0) == 1
    assert call(T=0) == 1


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", "/nonexistent/libmoe_b200.so")
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()


def test_backward_validation(lib):
    fake = ctypes.c_void_p(0x10000)
    s = B.make_shape(64, 256, 12, 4, 4, 128, "bf16")
    nb = lib.moe_backward_workspace_bytes(ctypes.byref(s))
    # status word + dlogits [T, E] + dau [T*K, 2I] (bf16)
    assert nb >= 256 + 64 * 16 * 2 + 64 * 4 * 2 * 128 * 2
    # bf16 backward needs d and I multiples of 128 and E multiple of 8
    for bad in (B.make_shape(64, 192, 12, 4, 4, 128, "bf16"),
                B.make_shape(64, 256, 12, 4, 4, 64, "bf16"),
                B.make_shape(64, 256, 12, 2, 4, 128, "bf16")):
        nbb = lib.moe_backward_workspace_bytes(ctypes.byref(bad))
        assert lib.moe_expert_ffn_backward(ctypes.byref(bad), fake, fake, fake, fake, fake, fake,
                                           fake, fake, fake, fake, fake, fake, fake, nbb,
                                           None) == 2
        assert lib.moe_route_backward(ctypes.byref(bad), fake, fake, fake, fake, fake, None, 0,
                                      0.0, 0, fake, fake, fake, nbb, None) == 2
    # workspace too small, NULL operand
    assert lib.moe_expert_ffn_backward(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake,
                                       fake, fake, fake, fake, fake, fake, nb - 256, None) == 3
    assert lib.moe_expert_ffn_backward(ctypes.byref(s), fake, fake, fake, fake, fake, fake, None,
                                       fake, fake, fake, fake, fake, fake, nb, None) == 1
    assert b"au" in lib.moe_last_error()
    assert lib.moe_combine_backward(ctypes.byref(s), fake, fake, fake, fake, fake, None, 1.0,
                                    fake, fake, None) == 1
    assert b"dout" in lib.moe_last_error()
    assert lib.moe_permute_backward(ctypes.byref(s), fake, fake, fake, fake, fake,
                                    ctypes.c_void_p(0x10004), 1.0, fake, None) == 1
    assert b"dx_router" in lib.moe_last_error()
    assert lib.moe_expert_gate_up_save(ctypes.byref(s), fake, fake, fake, fake, fake, None,
                                       fake, B.workspace_bytes(s), None) == 1


def test_route_backward_lb_validation(lib):
    fake = ctypes.c_void_p(0x10000)
    s = B.make_shape(64, 256, 12, 4, 4, 128, "bf16")
    nb = lib.moe_backward_workspace_bytes(ctypes.byref(s))
    # lb_groups must divide N, lb_tokens >= 1
    assert lib.moe_route_backward(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 5, 0.01,
                                  64, fake, fake, fake, nb, None) == 1
    assert b"lb_groups" in lib.moe_last_error()
    assert lib.moe_route_backward(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 4, 0.01,
                                  0, fake, fake, fake, nb, None) == 1


def test_pipeline_settings_validation(lib):
    assert lib.moe_debug_set_pipeline(61_000_000_000, 0) == 1  # above one minute
    assert b"above one minute" in lib.moe_last_error()
    assert lib.moe_debug_set_pipeline(1_000_000, 1) == 0
    assert lib.moe_debug_set_pipeline(0, 0) == 0  # back to the defaults
