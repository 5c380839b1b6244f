"""Host-side tests of the C ABI: the library builds and loads, exports every
symbol include/moe_capi.h declares, sizes its workspace, and rejects bad
arguments before launching anything (no GPU needed)."""

import ctypes
import os
import re

import pytest

import quantized_expert_ffn_moe_b200 as q
from quantized_expert_ffn_moe_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_capi.h")


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return q.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(moe_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("moe_route", "moe_layer_forward", "moe_stack_forward", "moe_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(q.EXPORTS) <= set(declared_functions())


FULL = dict(experts=512, hidden=2048, inter=768, top_k=10, shared=True, bits=4, block=32)


def cfg(**kw):
    d = dict(FULL)
    d.update(kw)
    return q.config_of(d["experts"], d["hidden"], d["inter"], d["top_k"], d["shared"], d["bits"], d["block"])


def test_workspace_bytes(lib):
    a = q.moe_workspace_bytes(cfg(), 1)
    b = q.moe_workspace_bytes(cfg(), 16)
    c = q.moe_workspace_bytes(cfg(), 4096)
    assert 0 < a < b < c
    # scratch at T=4096: h (fp32) + Y (fp32) + gathered X (bf16) dominate
    P = 4096 * 11
    assert c >= P * (768 * 4 + 2048 * 4 + 2048 * 2)
    assert q.moe_workspace_bytes(cfg(), 0) > 0
    assert q.moe_workspace_bytes(cfg(), -1) == 0


@pytest.mark.parametrize("kw", [dict(bits=3), dict(bits=4, block=16), dict(bits=4, block=64), dict(bits=2, block=32),
                                dict(bits=2, block=128), dict(hidden=300),
                                dict(experts=500), dict(top_k=17), dict(inter=100), dict(experts=2048)])
def test_unsupported_configs_report_zero_workspace(lib, kw):
    assert q.moe_workspace_bytes(cfg(**kw), 16) == 0


def test_tiny_and_2bit_configs_supported(lib):
    assert q.moe_workspace_bytes(q.config_of(64, 256, 128, 4, True, 4, 32), 8) > 0
    assert q.moe_workspace_bytes(cfg(bits=2, block=16), 64) > 0
    assert q.moe_workspace_bytes(cfg(shared=False), 64) > 0
    assert q.moe_workspace_bytes(cfg(bits=4, block=128), 64) > 0      # GPTQ-style 128-element groups


ROW_SCALES = ("gate_up_row_scales", "down_row_scales", "shared_gate_up_row_scales", "shared_down_row_scales")


def _fake_weights(shared=True, misalign=None, fp8=False):
    # addresses are never dereferenced on these paths
    base = 1 << 20
    w = q._Weights()
    for i, (name, _) in enumerate(q._Weights._fields_):
        setattr(w, name, base * (i + 1))
    if not shared:
        for n in ("shared_gate_up_codes", "shared_gate_up_scales", "shared_down_codes", "shared_down_scales",
                  "shared_gate_up_row_scales", "shared_down_row_scales"):
            setattr(w, n, None)
    if not fp8:
        for n in ROW_SCALES:
            setattr(w, n, None)
    w.router_bias = None
    w.shared_gate_w = None
    if misalign:
        setattr(w, misalign, getattr(w, misalign) + 8)
    return w


def _layer(lib, c, w, x=1 << 30, T=4, y=2 << 30, ws=3 << 30, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.moe_workspace_bytes(ctypes.byref(c), T)
    return lib.moe_layer_forward(ctypes.byref(c), ctypes.byref(w), x, T, y, ws, ws_bytes, None)


def test_fp8_scale_arguments(lib):
    """scale_fmt 1 needs the fp32 row scales (16-byte aligned), scale_fmt 0
    refuses them; fp8 scales only with blocks of 32 (4-bit) / 16 (2-bit)."""
    c8 = cfg()
    c8.scale_fmt = 1
    assert lib.moe_workspace_bytes(ctypes.byref(c8), 16) > 0
    assert _layer(lib, c8, _fake_weights(fp8=True), ws_bytes=100) == -3     # arguments pass, workspace too small
    w = _fake_weights(fp8=False)
    assert _layer(lib, c8, w) == -1                                        # row scales missing
    w = _fake_weights(fp8=True)
    w.down_row_scales += 2
    assert _layer(lib, c8, w) == -1                                        # misaligned row scales
    w = _fake_weights(fp8=True)
    w.shared_gate_up_row_scales += 4
    assert _layer(lib, c8, w) == -1                                        # 4-byte but not 16-byte aligned
    w = _fake_weights(fp8=True, shared=False)
    c8s = cfg(shared=False)
    c8s.scale_fmt = 1
    assert _layer(lib, c8s, w, ws_bytes=100) == -3                         # no shared expert: no shared row scales
    assert _layer(lib, cfg(), _fake_weights(fp8=True)) == -1               # fp16 scales with row scales
    c2 = cfg()
    c2.scale_fmt = 2
    assert lib.moe_workspace_bytes(ctypes.byref(c2), 16) == 0
    cg = cfg(bits=4, block=128)
    cg.scale_fmt = 1
    assert lib.moe_workspace_bytes(ctypes.byref(cg), 16) == 0
    ch = cfg()
    ch.scale_fmt = 1
    ch.half_levels = 1
    assert lib.moe_workspace_bytes(ctypes.byref(ch), 16) == 0


def test_layer_forward_argument_errors(lib):
    c = cfg()
    w = _fake_weights()
    assert _layer(lib, c, w, T=0) == 0                       # empty batch: no-op
    assert _layer(lib, c, w, T=-1) == q.MOE_OK - 1           # MOE_ERR_INVALID_ARG
    assert _layer(lib, c, w, x=None) == -1
    assert _layer(lib, c, w, x=(1 << 30) + 2) == -1          # misaligned x
    assert _layer(lib, c, w, y=(1 << 30) + 1024) == -1       # y overlaps x
    assert _layer(lib, c, w, ws=(3 << 30) + 16) == -1        # workspace not 256-aligned
    assert _layer(lib, c, w, ws_bytes=100) == -3             # MOE_ERR_WORKSPACE
    assert _layer(lib, c, _fake_weights(misalign="down_codes")) == -1
    assert _layer(lib, c, _fake_weights(shared=False)) == -1  # shared expert configured but missing
    assert _layer(lib, cfg(shared=False), _fake_weights(shared=False), ws_bytes=0) == -3
    assert _layer(lib, cfg(bits=3), w) == -2                  # MOE_ERR_UNSUPPORTED
    g = _fake_weights()
    g.shared_gate_w = 1 << 24
    assert _layer(lib, cfg(), g, ws_bytes=0) == -3           # a gate with a shared expert is valid
    assert _layer(lib, cfg(shared=False), g) == -1           # a gate needs a shared expert
    g.shared_gate_w = (1 << 24) + 8
    assert _layer(lib, cfg(), g) == -1                        # misaligned gate vector
    assert lib.moe_layer_forward(None, ctypes.byref(w), 1 << 30, 4, 2 << 30, 3 << 30, 1 << 40, None) == -1


def test_noalloc_argument_errors_match_layer_forward(lib):
    """The allocation-free entry point checks its arguments in the same order
    as moe_layer_forward (the size limit of its fixed scratch takes the place
    of the workspace check), so it reports the same codes, all on the host."""
    c = cfg()
    w = _fake_weights()

    def na(c, w, x=1 << 30, T=4, y=2 << 30):
        return lib.moe_layer_forward_noalloc(ctypes.byref(c), ctypes.byref(w) if w is not None else None, x, T, y,
                                             None)
    assert na(c, w, T=0) == 0                                  # empty batch: no-op
    assert na(c, w, T=-1) == -1
    assert na(c, None, T=24) == -1                             # null weights beat the size limit
    assert na(c, w, x=None, T=1000) == -1                      # null x beats the size limit
    assert na(c, w, y=(1 << 30) + 1024) == -1                  # y overlaps x
    assert na(cfg(bits=3), w) == -2                             # the config's own code (unsupported)
    assert na(cfg(top_k=0), w) == -1                            # ... or invalid
    assert na(c, _fake_weights(misalign="down_codes")) == -1
    assert na(c, w, T=24) == -3                                 # beyond the 4 MiB scratch: MOE_ERR_WORKSPACE
    assert lib.moe_noalloc_device_status(None) == -1


def _layer_ep(lib, c, w, rank, size, x=1 << 30, T=4, y=2 << 30, ws=3 << 30, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.moe_workspace_bytes(ctypes.byref(c), T)
    return lib.moe_layer_forward_ep(ctypes.byref(c), ctypes.byref(w), x, T, rank, size, y, ws, ws_bytes, None)


def test_layer_forward_ep_argument_errors(lib):
    """Rejections happen on the host, before any launch."""
    c = cfg()
    w = _fake_weights()
    E = c.num_experts
    assert _layer_ep(lib, c, w, 0, 2, T=0) == 0                  # empty batch: no-op
    assert _layer_ep(lib, c, w, 0, 0) == -1                      # ep_size < 1
    assert _layer_ep(lib, c, w, 2, 2) == -1                      # rank out of range
    assert _layer_ep(lib, c, w, -1, 2) == -1
    assert _layer_ep(lib, c, w, 0, E + 1) == -1                  # more ranks than experts
    assert _layer_ep(lib, c, w, 0, 2, y=None) == -1
    assert _layer_ep(lib, c, w, 0, 2, y=(2 << 30) + 8) == -1     # misaligned fp32 output
    assert _layer_ep(lib, c, w, 0, 2, y=(1 << 30) + 4096) == -1  # output overlaps x
    assert _layer_ep(lib, c, w, 0, 2, ws_bytes=100) == -3
    # the shared expert is required on rank 0 only
    assert _layer_ep(lib, c, _fake_weights(shared=False), 0, 2) == -1
    assert _layer_ep(lib, c, _fake_weights(shared=False), 1, 2, ws_bytes=0) == -3
    assert _layer_ep(lib, cfg(bits=3), w, 0, 2) == -2
    assert lib.moe_layer_forward_ep(ctypes.byref(c), None, 1 << 30, 4, 0, 2, 2 << 30, 3 << 30, 1 << 30, None) == -1


def test_wait_probe_argument_errors(lib):
    assert lib.moe_debug_wait_probe(None, None) == -1
    assert lib.moe_debug_wait_probe((1 << 30) + 16, None) == -1


def test_route_and_stack_argument_errors(lib):
    c = cfg()
    n = lib.moe_workspace_bytes(ctypes.byref(c), 4)
    assert lib.moe_route(ctypes.byref(c), 1 << 20, None, 1 << 30, 0, 1 << 31, 1 << 32, None, None, None,
                         3 << 30, n, None) == 0
    assert lib.moe_route(ctypes.byref(c), None, None, 1 << 30, 4, 1 << 31, 1 << 32, None, None, None,
                         3 << 30, n, None) == -1
    assert lib.moe_route(ctypes.byref(c), 1 << 20, None, 1 << 30, 4, None, 1 << 32, None, None, None,
                         3 << 30, n, None) == -1
    arr = (q._Weights * 2)(_fake_weights(), _fake_weights(misalign="router_w"))
    assert lib.moe_stack_forward(ctypes.byref(c), arr, 2, 1 << 30, 4, None, 3 << 30, n, None) == -1
    assert lib.moe_stack_forward(ctypes.byref(c), arr, 0, 1 << 30, 4, None, 3 << 30, n, None) == 0
    assert lib.moe_stack_forward(ctypes.byref(c), arr, 1, 1 << 30, 0, None, 3 << 30, n, None) == 0
    assert lib.moe_dequant_rows(ctypes.byref(cfg(bits=3)), 1 << 20, 1 << 21, 0, 1, 256, 1 << 22, None) == -2


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert q.moe_status_str(s) and q.moe_status_str(s) != "unknown status"
    assert q.moe_status_str(42) == "unknown status"


def test_binding_fails_loudly_without_library(tmp_path):
    import importlib
    mod = importlib.import_module("quantized_expert_ffn_moe_b200")
    with pytest.raises(RuntimeError):
        mod._lib, saved = None, mod._lib
        try:
            mod.load_library(str(tmp_path / "missing.so"))
        finally:
            mod._lib = saved


def test_header_is_plain_c(tmp_path):
    """The boundary header compiles as C99 (no C++ in the interface) and a C
    caller can name every entry point with the declared types."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_capi.c"
    src.write_text("""
#include "moe_capi.h"
int use(void* ws, size_t n, const uint16_t* x, uint16_t* y, float* yp, void* stream) {
  moe_config c = {512, 2048, 768, 10, 768, 4, 32};
  moe_layer_weights w = {0};
  int32_t code = 0;
  size_t need = moe_workspace_bytes(&c, 16);
  int st = moe_layer_forward(&c, &w, x, 16, y, ws, n, stream);
  st |= moe_layer_forward_ep(&c, &w, x, 16, 0, 2, yp, ws, n, stream);
  st |= moe_stack_forward(&c, &w, 1, y, 16, NULL, ws, n, stream);
  st |= moe_device_status(ws, &code);
  st |= moe_layer_forward_noalloc(&c, &w, x, 16, y, stream);
  st |= moe_noalloc_device_status(&code);
  moe_debug_decode_path(0);
  (void)moe_status_str(st);
  return st + (int)need + code;
}
""")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I", inc, str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_null_arguments_are_rejected_everywhere(lib):
    """Every entry point turns NULL pointers into MOE_ERR_INVALID_ARG on the
    host, without touching the device."""
    c = cfg()
    w = _fake_weights()
    n = lib.moe_workspace_bytes(ctypes.byref(c), 4)
    assert lib.moe_workspace_bytes(None, 4) == 0
    assert lib.moe_route(None, 1 << 20, None, 1 << 30, 4, 1 << 31, 1 << 32, None, None, None, 3 << 30, n, None) == -1
    assert lib.moe_layer_forward(ctypes.byref(c), None, 1 << 30, 4, 2 << 30, 3 << 30, n, None) == -1
    assert lib.moe_layer_forward(ctypes.byref(c), ctypes.byref(w), 1 << 30, 4, 2 << 30, None, n, None) == -1
    assert lib.moe_layer_forward_ep(None, ctypes.byref(w), 1 << 30, 4, 0, 2, 2 << 30, 3 << 30, n, None) == -1
    assert lib.moe_stack_forward(ctypes.byref(c), None, 1, 1 << 30, 4, None, 3 << 30, n, None) == -1
    assert lib.moe_stack_forward(None, None, 1, 1 << 30, 4, None, 3 << 30, n, None) == -1
    arr = (q._Weights * 1)(_fake_weights())
    assert lib.moe_stack_forward(ctypes.byref(c), arr, 1, None, 4, None, 3 << 30, n, None) == -1
    assert lib.moe_device_status(None, None) == -1
    assert lib.moe_dequant_rows(None, 1 << 20, 1 << 21, 0, 1, 256, 1 << 22, None) == -1
    assert lib.moe_dequant_rows(ctypes.byref(c), None, 1 << 21, 0, 1, 256, 1 << 22, None) == -1
    assert lib.moe_layer_forward_noalloc(None, ctypes.byref(w), 1 << 30, 4, 2 << 30, None) == -1
    assert lib.moe_profile_end(None, None) == -1
