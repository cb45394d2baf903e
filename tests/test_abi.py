"""C ABI checks that need no GPU: the library builds, loads, exports every
function include/gptblock.h declares, sizes workspaces on the host and
rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def gb():
    from gpt_transformer_block_b200 import build
    build.build()
    import gpt_transformer_block_b200 as gb
    gb.load()
    return gb


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gptblock.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"^\s*typedef[^;]*;", "", text, flags=re.M)  # callback types are not functions
    names = re.findall(r"^\s*(?:const\s+)?(?:long\s+long|unsigned\s+long\s+long|[A-Za-z_]\w*)\s*\*?\s*"
                       r"([A-Za-z_]\w*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("gpt_block_forward", "gpt_block_backward", "gpt_stack_step", "lm_head_xent"):
        assert n in names


def test_library_exports_every_declared_symbol(gb):
    lib = gb.load()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(gb.EXPORTS) <= set(declared_functions())


def test_error_strings(gb):
    lib = gb.load()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.gptb_error_string(code)


def test_workspace_sizes_scale_with_tokens(gb):
    c = synth.config("d24", B=1, T=256, n_layer=2)
    cfg = gb.make_config(c)
    saved = gb.gptb_workspace_bytes(cfg, gb.WS_BLOCK_SAVED)
    # h, h2 [N,d] + qkv [N,3d] + o [N,d] + act [N,4d] in bf16, plus fp32 row stats
    # (u is not kept: the ReLU^2 backward uses 2 sqrt(act) = 2 relu(u))
    N, d = 256, 1536
    assert saved >= 2 * N * (d + 3 * d + d + d + 4 * d)
    c2 = synth.config("d24", B=2, T=256, n_layer=2)
    saved2 = gb.gptb_workspace_bytes(gb.make_config(c2), gb.WS_BLOCK_SAVED)
    assert 1.9 * saved < saved2 < 2.1 * saved
    stack = gb.gptb_workspace_bytes(cfg, gb.WS_STACK)
    assert stack > 2 * saved
    assert gb.gptb_workspace_bytes(cfg, 99) == 0


def _f32_cfg(gb, **kw):
    c = synth.config("block_fp32", **kw)
    return gb.make_config(c)


def test_null_pointers_rejected_without_device_work(gb):
    lib = gb.load()
    cfg = _f32_cfg(gb)
    w = gb.BlockWeights()
    rc = lib.gpt_block_forward(ctypes.byref(cfg), 0, ctypes.byref(w), None, None, None, None, None, None, None)
    assert rc == gb.ERR_INVALID_ARG
    rc = lib.gpt_block_forward(None, 0, ctypes.byref(w), None, None, None, None, None, None, None)
    assert rc == gb.ERR_INVALID_ARG
    rc = lib.gpt_stack_step(ctypes.byref(cfg), None, None, None, None, None, None, None)
    assert rc == gb.ERR_INVALID_ARG


def test_bad_shapes_rejected(gb):
    lib = gb.load()
    w = gb.BlockWeights()
    for bad in (dict(n_kv_head=3), dict(d=100), dict(n_layer=0), dict(head_dim=7), dict(T=2048),
                dict(backout_layer=5), dict(mlp_hidden=100)):
        cfg = _f32_cfg(gb, **bad)
        rc = lib.gpt_block_forward(ctypes.byref(cfg), 0, ctypes.byref(w), None, None, None, None, None, None, None)
        assert rc in (gb.ERR_INVALID_ARG, gb.ERR_UNSUPPORTED), bad


def test_unknown_dtype_unsupported(gb):
    lib = gb.load()
    cfg = _f32_cfg(gb)
    cfg.dtype = 7
    w = gb.BlockWeights()
    assert lib.gpt_block_forward(ctypes.byref(cfg), 0, ctypes.byref(w), None, None, None, None, None, None,
                                 None) == gb.ERR_UNSUPPORTED


def test_optimizer_entry_points_validate_on_the_host(gb):
    lib = gb.load()
    # workspace: 0 for bad shapes, grows with the matrix and the Gram side
    assert gb.gptb_polar_express_workspace_bytes(0, 8, 2) == 0
    assert gb.gptb_polar_express_workspace_bytes(8, 8, 0) == 0
    assert gb.gptb_polar_express_workspace_bytes(8, 8, 65) == 0
    small = gb.gptb_polar_express_workspace_bytes(64, 32, 5)
    assert small >= 1024 + 2 * 64 * 32 * 2 + 2 * 32 * 32 * 2
    assert gb.gptb_polar_express_workspace_bytes(32, 64, 5) == small  # wide: same buffers
    coeffs = (ctypes.c_float * 3)(1.5, -0.5, 0.0)
    # shapes that are not multiples of 8, bad step counts and null pointers are rejected before any CUDA call
    for m, n, steps in ((12, 8, 1), (8, 12, 1), (8, 8, 0), (8, 8, 65)):
        assert lib.gptb_polar_express(16, 4096, m, n, coeffs, steps, 256, 1 << 20, None) == gb.ERR_INVALID_ARG
    assert lib.gptb_polar_express(None, 4096, 8, 8, coeffs, 1, 256, 1 << 20, None) == gb.ERR_INVALID_ARG
    # out overlapping G
    assert lib.gptb_polar_express(4096, 4096 + 64, 8, 8, coeffs, 1, 256, 1 << 20, None) == gb.ERR_INVALID_ARG
    # too small a workspace
    assert lib.gptb_polar_express(4096, 1 << 16, 8, 8, coeffs, 1, 256, 16, None) == gb.ERR_WORKSPACE
    # AdamW: null arrays, negative n, step 0, beta outside [0, 1)
    assert lib.gptb_adamw_step(None, 16, 32, 48, None, 4, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == gb.ERR_INVALID_ARG
    assert lib.gptb_adamw_step(16, 16, 32, 48, None, -1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == gb.ERR_INVALID_ARG
    assert lib.gptb_adamw_step(16, 16, 32, 48, None, 4, 1e-3, 0.9, 0.999, 1e-8, 0.0, 0, None) == gb.ERR_INVALID_ARG
    assert lib.gptb_adamw_step(16, 16, 32, 48, None, 4, 1e-3, 1.0, 0.999, 1e-8, 0.0, 1, None) == gb.ERR_INVALID_ARG
    assert lib.gptb_adamw_step(16, 16, 32, 48, None, 0, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == gb.OK
