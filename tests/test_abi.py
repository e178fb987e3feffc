"""Host-side checks of the C ABI library: it loads, exports every declared
entry point, sizes workspaces, and refuses bad arguments before any launch.
No GPU is touched."""
import ctypes
import os
import re

import pytest
import torch

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moeffn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(\w+)\s*\([^;{]*\)\s*;", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_library_builds_and_loads():
    import moe_expert_layer_dequant_b200 as lib
    assert os.path.exists(lib.LIB_PATH)


def test_every_declared_symbol_is_exported():
    import moe_expert_layer_dequant_b200 as lib
    names = declared_functions()
    assert "ffn_dense" in names and "moe_layer" in names and "moe_router_topk" in names
    assert "ffn_shared_expert" in names and len(names) >= 11
    so = ctypes.CDLL(lib.LIB_PATH)
    missing = [n for n in names if not hasattr(so, n)]
    assert not missing, missing


def test_workspace_sizes():
    import moe_expert_layer_dequant_b200 as lib
    d1 = lib.workspace_bytes(lib.KIND_DENSE, 1, 4096, 14336)
    d16 = lib.workspace_bytes(lib.KIND_DENSE, 16, 4096, 14336)
    assert 0 < d1 < d16
    # activations [M][I] bf16 + fp32 K-split partials [S][M][H], S >= 1
    assert d16 >= 16 * 14336 * 2 + 16 * 4096 * 4
    assert lib.workspace_bytes(lib.KIND_MOE, 4, 2048, 768, 128, 8) > 0
    assert lib.workspace_bytes(lib.KIND_DENSE, 0, 4096, 14336) == 0
    assert lib.workspace_bytes(99, 1, 4096, 14336) == 0


# Pointer-free refusals: every call below must fail validation before any
# CUDA call. They use fake addresses, so they only run where no GPU exists.
nogpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake-pointer refusals run only without a GPU")


def _fake_qweight(lib, fmt, rows, cols, base):
    return lib._QWeight(fmt, rows, cols, base, base + 0x100000, base + 0x200000 if fmt == lib.Q_INT4_AFFINE_G32 else None)


def _fake_ffn(lib, fmt, H, I):
    return lib._FFN(_fake_qweight(lib, fmt, I, H, 0x10000000), _fake_qweight(lib, fmt, I, H, 0x20000000),
                    _fake_qweight(lib, fmt, H, I, 0x30000000))


@nogpu
def test_refusals_before_launch():
    import moe_expert_layer_dequant_b200 as lib
    L = lib._lib
    f = _fake_ffn(lib, lib.Q_INT4_AFFINE_G32, 256, 512)
    x, r, ws = 0x40000000, 0x50000000, 0x60000000
    need = lib.workspace_bytes(lib.KIND_DENSE, 2, 256, 512)
    assert L.ffn_dense(None, x, r, 2, 0, ws, need, None) == -1
    assert L.ffn_dense(ctypes.byref(f), x, r, 0, 0, ws, need, None) == -1          # M = 0
    assert L.ffn_dense(ctypes.byref(f), x, r, 2, 7, ws, need, None) == -1          # bad act
    assert L.ffn_dense(ctypes.byref(f), x, x, 2, 0, ws, need, None) == -1          # x aliases residual
    assert L.ffn_dense(ctypes.byref(f), x + 2, r, 2, 0, ws, need, None) == -1      # misaligned x
    assert L.ffn_dense(ctypes.byref(f), x, r, 2, 0, None, need, None) == -3        # no workspace
    assert L.ffn_dense(ctypes.byref(f), x, r, 2, 0, ws, need - 1, None) == -3      # too small
    assert L.ffn_dense(ctypes.byref(f), x, r, 2, 0, ws + 16, need, None) == -3     # misaligned workspace
    assert b"workspace" in L.moeffn_last_error()
    bad = _fake_ffn(lib, lib.Q_INT4_AFFINE_G32, 256 + 16, 512)                      # K % 32 != 0
    assert L.ffn_dense(ctypes.byref(bad), x, r, 2, 0, ws, 1 << 30, None) == -1
    fmt = _fake_ffn(lib, 9, 256, 512)                                                # unknown format
    assert L.ffn_dense(ctypes.byref(fmt), x, r, 2, 0, ws, 1 << 30, None) == -2
    # block types are per tensor, but gate and up share one fused kernel
    mixed = _fake_ffn(lib, lib.Q_INT4_AFFINE_G32, 256, 512)
    mixed.up = _fake_qweight(lib, lib.Q_INT8_ROW, 512, 256, 0x30000000)
    assert L.ffn_dense(ctypes.byref(mixed), x, r, 2, 0, ws, 1 << 30, None) == -2
    assert b"gate and up" in L.moeffn_last_error()
    unal = _fake_ffn(lib, lib.Q_INT4_AFFINE_G32, 256, 512)
    unal.down = lib._QWeight(lib.Q_INT4_AFFINE_G32, 256, 512, 0x30000000, 0x30100002, 0x30200000)   # scale + 2 bytes
    assert L.ffn_dense(ctypes.byref(unal), x, r, 2, 0, ws, 1 << 30, None) == -1
    assert b"16-byte" in L.moeffn_last_error()
    huge = _fake_ffn(lib, lib.Q_INT8_ROW, 65536, 512)                                 # stages do not fit
    assert L.ffn_dense(ctypes.byref(huge), x, r, 2, 0, ws, 1 << 40, None) == -2
    q4k = _fake_ffn(lib, lib.Q_Q4_K, 256 + 128, 512)                                 # Q4_K: K % 256 != 0
    assert L.ffn_dense(ctypes.byref(q4k), x, r, 2, 0, ws, 1 << 30, None) == -1
    assert b"256" in L.moeffn_last_error()
    q4k = _fake_ffn(lib, lib.Q_Q4_K, 256, 512)
    q4k.gate.q = 0x10000008                                                          # misaligned blocks
    assert L.ffn_dense(ctypes.byref(q4k), x, r, 2, 0, ws, 1 << 30, None) == -1
    shape = _fake_ffn(lib, lib.Q_INT8_ROW, 256, 512)
    shape.down = _fake_qweight(lib, lib.Q_INT8_ROW, 512, 256, 0x30000000)           # transposed down
    assert L.ffn_dense(ctypes.byref(shape), x, r, 2, 0, ws, 1 << 30, None) == -1
    assert b"shape" in L.moeffn_last_error()


@nogpu
def test_router_and_plan_refusals():
    import moe_expert_layer_dequant_b200 as lib
    L = lib._lib
    router = lib._QWeight(lib.F32, 8, 256, 0x10000000, None, None)
    x, ws = 0x40000000, 0x60000000
    idx, w = 0x70000000, 0x71000000
    assert L.moe_router_topk(ctypes.byref(router), x, 4, 0, None, idx, w, None, None, ws, 1 << 20, None) == -2
    assert L.moe_router_topk(ctypes.byref(router), x, 4, 9, None, idx, w, None, None, ws, 1 << 20, None) == -2
    assert L.moe_router_topk(ctypes.byref(router), x, 4, 2, None, idx, w, 0x72000000, None, ws, 1 << 20, None) == -1
    int8_router = lib._QWeight(lib.Q_INT8_ROW, 8, 256, 0x10000000, 0x11000000, None)
    assert L.moe_router_topk(ctypes.byref(int8_router), x, 4, 2, None, idx, w, None, None, ws, 1 << 20, None) == -2
    # The routed path takes INT4-affine experts only (refuse, do not degrade).
    experts = (lib._FFN * 8)(*[_fake_ffn(lib, lib.Q_INT8_ROW, 256, 512) for _ in range(8)])
    desc = lib._MoeDesc(8, 2, 0, router, experts, None, None)
    h = ctypes.c_void_p()
    assert L.moe_plan_create(ctypes.byref(desc), ctypes.byref(h)) == -2
    assert b"INT4" in L.moeffn_last_error()
    q4k_experts = (lib._FFN * 8)(*[_fake_ffn(lib, lib.Q_Q4_K, 256, 512) for _ in range(8)])
    assert L.moe_plan_create(ctypes.byref(lib._MoeDesc(8, 2, 0, router, q4k_experts, None, None)), ctypes.byref(h)) == -2
    desc.top_k = 0
    assert L.moe_plan_create(ctypes.byref(desc), ctypes.byref(h)) == -2
    assert L.moe_layer(None, x, 0x50000000, 1, None, ws, 1 << 20, None) == -1
    # Gemma form: the shared branch's post-norm needs a shared expert and excludes its gate.
    experts4 = (lib._FFN * 8)(*[_fake_ffn(lib, lib.Q_INT4_AFFINE_G32, 256, 512) for _ in range(8)])
    shared = _fake_ffn(lib, lib.Q_INT4_AFFINE_G32, 256, 512)
    gate = lib._QWeight(lib.BF16, 1, 256, 0x12000000, None, None)
    desc = lib._MoeDesc(8, 2, 0, router, experts4, None, None, None, 0x13000000, 1e-6)
    assert L.moe_plan_create(ctypes.byref(desc), ctypes.byref(h)) == -1
    desc = lib._MoeDesc(8, 2, 0, router, experts4, ctypes.pointer(shared), ctypes.pointer(gate), None, 0x13000000, 1e-6)
    assert L.moe_plan_create(ctypes.byref(desc), ctypes.byref(h)) == -1
    assert b"shared_gate" in L.moeffn_last_error()
    assert L.moe_layer_prenorm(None, 0x13000000, 1e-6, 0x50000000, 1, None, ws, 1 << 20, None) == -1
    f = _fake_ffn(lib, lib.Q_INT4_AFFINE_G32, 256, 512)
    assert L.ffn_dense_prenorm(ctypes.byref(f), None, 1e-6, 0x50000000, 2, 0, ws, 1 << 30, None) == -1


def test_fault_injection_export_validates_on_the_host():
    """The failure-injection test export refuses unknown kinds, depths outside
    1..8 and wait limits outside 1 us..1 s before any launch (host only)."""
    import moe_expert_layer_dequant_b200 as lib
    for args in ((3, 0, 10), (2, 9, 10), (2, 0, 10), (1, -1, 10), (1, 0, 0), (1, 0, 2000000)):
        with pytest.raises(lib.MoeffnError) as e:
            lib.test_inject_gemv_fault(*args)
        assert e.value.status == -1
    lib.test_inject_gemv_fault(0)                  # cancel: always accepted


@nogpu
def test_expert_parallel_refusals():
    """moe_dispatch_rows, moe_experts_grouped and moe_combine validate on the
    host before any launch; workspace queries size the combine's inverse map."""
    import moe_expert_layer_dequant_b200 as lib
    L = lib._lib
    x, idx, perm, rows, exp = 0x40000000, 0x41000000, 0x42000000, 0x43000000, 0x44000000
    assert L.moe_dispatch_rows(None, idx, perm, 4, 2, 256, rows, exp, None) == -1
    assert L.moe_dispatch_rows(x, idx, perm, 0, 2, 256, rows, exp, None) == -1       # M = 0
    assert L.moe_dispatch_rows(x, idx, perm, 4, 0, 256, rows, exp, None) == -1       # top_k = 0
    assert L.moe_dispatch_rows(x, idx, perm, 4, 17, 256, rows, exp, None) == -1      # top_k above 16
    assert L.moe_dispatch_rows(x, idx, perm, 4, 2, 260, rows, exp, None) == -1       # H % 8 != 0
    assert L.moe_dispatch_rows(x + 2, idx, perm, 4, 2, 256, rows, exp, None) == -1   # misaligned x
    assert b"aligned" in L.moeffn_last_error()
    assert L.moe_experts_grouped(None, rows, 8, exp, 0, 0x45000000, 0x60000000, 1 << 20, None) == -1
    assert L.moe_experts_workspace_bytes(None, 8) == 0
    d, w, res, sd, ws = 0x46000000, 0x47000000, 0x48000000, 0x49000000, 0x60000000
    need = L.moe_combine_workspace_bytes(4, 2)
    assert need >= 4 * 2 * 4 and L.moe_combine_workspace_bytes(0, 2) == 0
    assert L.moe_combine(None, perm, w, 4, 2, 256, None, None, res, ws, need, None) == -1
    assert L.moe_combine(d, perm, w, 4, 2, 256, sd, None, res, ws, need, None) == -1   # shared_d without its gate
    assert b"gate_logit" in L.moeffn_last_error()
    assert L.moe_combine(d, perm, w, 0, 2, 256, None, None, res, ws, need, None) == -1  # M = 0
    assert L.moe_combine(d, perm, w, 4, 2, 258, None, None, res, ws, need, None) == -1  # H % 4 != 0
    assert L.moe_combine(d + 4, perm, w, 4, 2, 256, None, None, res, ws, need, None) == -1
    assert L.moe_combine(d, perm, w, 4, 2, 256, None, None, res, ws, need - 1, None) == -3
