"""The C ABI library loads without a GPU, exports every entry point that
include/*.h declares, and rejects bad arguments on the host (these calls
return before any CUDA call is made)."""
import glob
import os
import re

import pytest

from video_diffusion_transformer_fwd_b200 import build_lib, wan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_lib.build(verbose=False)
    return wan.load()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(wan_[a-z0-9_]+)\s*\(",
                            src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("wan_rope_freqs", "wan_block_forward", "wan_attention", "wan_euler_cfg_step",
              "wan_block_workspace_bytes", "wan_last_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_binding_has_the_c_names():
    for n in declared_functions():
        assert callable(getattr(wan, n)), n


def dims(**kw):
    base = dict(F=2, H=4, W=4, dim=128, heads=4, ffn_dim=512, text_len=8, eps=1e-6, dtype="f32")
    base.update(kw)
    return wan.make_dims(**base)


def test_workspace_size_and_offsets(lib):
    d = dims()
    n = wan.wan_block_workspace_bytes(d, 2)
    assert n > 0
    offs = [wan.wan_block_workspace_offset(d, 2, i) for i in range(9)]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    L, D = 32, 128
    # qkv buffer holds [B*L, 3D] fp32
    assert offs[wan.WAN_WS_QKV] - offs[wan.WAN_WS_ACT] >= 2 * L * D * 4
    assert offs[wan.WAN_WS_O] - offs[wan.WAN_WS_QKV] >= 2 * L * 3 * D * 4
    assert wan.wan_block_workspace_offset(d, 2, 99) == (1 << 64) - 1
    # bf16 halves the activation buffers
    assert wan.wan_block_workspace_bytes(dims(dtype="bf16", dim=512, heads=4, ffn_dim=512), 1) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(dim=100), wan.WAN_EINVAL),
    (dict(heads=3), wan.WAN_EINVAL),
    (dict(ffn_dim=500), wan.WAN_EINVAL),
    (dict(F=0), wan.WAN_EINVAL),
    (dict(dtype=7), wan.WAN_EUNSUPPORTED),
    (dict(dtype="bf16"), wan.WAN_EUNSUPPORTED),       # head_dim 32 in bf16
    (dict(heads=1), wan.WAN_EUNSUPPORTED),            # fp32 head_dim 128 is fine -> see below
])
def test_block_forward_rejects_bad_dims(lib, kw, code):
    d = dims(**kw)
    if kw == dict(heads=1):
        d = dims(heads=1, dim=128 * 3)               # head_dim 384: unsupported
    w = wan.wan_block_weights()
    rc = wan.wan_block_forward(d, 1, 16, 16, None, 16, w, 16, 1024, 16, 1 << 30, None)
    assert rc == code
    assert wan.last_error() != ""
    assert wan.wan_block_workspace_bytes(d, 1) == 0


def test_block_forward_rejects_null_and_misaligned(lib):
    d = dims()
    w = wan.wan_block_weights()
    assert wan.wan_block_forward(d, 1, 16, 16, None, 16, w, 16, 1024, 16, 1 << 30, None) == wan.WAN_EINVAL
    w = wan.wan_block_weights(*([4096] * len(wan.WEIGHT_FIELDS)))
    assert wan.wan_block_forward(d, 1, 17, 16, None, 16, w, 16, 1024, 16, 1 << 30, None) == wan.WAN_EALIGN
    # rope table shorter than the grid
    assert wan.wan_block_forward(d, 1, 16, 16, None, 16, w, 16, 3, 16, 1 << 30, None) == wan.WAN_EINVAL
    # workspace too small
    assert wan.wan_block_forward(d, 1, 16, 16, None, 16, w, 16, 1024, 16, 100, None) == wan.WAN_EINVAL
    # B = 0 is an empty call
    assert wan.wan_block_forward(d, 0, 16, 16, None, 16, w, 16, 1024, 16, 0, None) == wan.WAN_OK


def test_other_entry_points_reject_bad_arguments(lib):
    assert wan.wan_rope_freqs(127, 1024, 1e4, 16, None) == wan.WAN_EINVAL
    assert wan.wan_rope_freqs(128, 0, 1e4, 16, None) == wan.WAN_EINVAL
    assert wan.wan_rope_freqs(128, 1024, 1e4, 8, None) == wan.WAN_EALIGN
    assert wan.wan_attention(1, 2, 8, 8, 96, wan.WAN_F32, 16, 32, 48, 64, None, 0.0, None, None, 0, None) == wan.WAN_EUNSUPPORTED
    assert wan.wan_attention(1, 2, 8, 8, 64, wan.WAN_BF16, 16, 32, 48, 64, None, 0.0, None, None, 0, None) == wan.WAN_EUNSUPPORTED
    assert wan.wan_attention(1, 2, 8, 8, 64, wan.WAN_F32, 16, 16 + 4096, 16 + 8192, 16, None, 0.0, None, None, 0, None) == wan.WAN_EINVAL
    # grid that does not match L
    assert wan.wan_attention(1, 2, 8, 8, 64, wan.WAN_F32, 1 << 20, 1 << 21, 1 << 22, 1 << 23, None, 0.0,
                             (1, 2, 3), 16, 1024, None) == wan.WAN_EINVAL
    assert wan.wan_attention(0, 2, 8, 8, 64, wan.WAN_F32, 16, 32, 48, 64, None, 0.0, None, None, 0, None) == wan.WAN_OK
    assert wan.wan_euler_cfg_step(16, 32, None, wan.WAN_F32, 0, 5.0, 0.9, 0.875, None) == wan.WAN_OK
    assert wan.wan_euler_cfg_step(None, 32, None, wan.WAN_F32, 10, 5.0, 0.9, 0.875, None) == wan.WAN_EINVAL
    assert wan.wan_euler_cfg_step(16, 32, None, 5, 10, 5.0, 0.9, 0.875, None) == wan.WAN_EUNSUPPORTED
    assert wan.wan_euler_cfg_step(18, 32, None, wan.WAN_F32, 10, 5.0, 0.9, 0.875, None) == wan.WAN_EALIGN


def test_noalloc_array_size_matches_header():
    """The binding's copy of WAN_NOALLOC_WORKSPACE_BYTES is the header's."""
    src = open(os.path.join(ROOT, "include", "wan.h")).read()
    m = re.search(r"#define\s+WAN_NOALLOC_WORKSPACE_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "define not found"
    assert int(m.group(1)) << int(m.group(2)) == wan.WAN_NOALLOC_WORKSPACE_BYTES


def test_noalloc_empty_and_invalid_calls_match_the_workspace_entry_point(lib):
    """B == 0 and invalid dims give wan_block_forward's status and message."""
    w = wan.wan_block_weights(*([4096] * len(wan.WEIGHT_FIELDS)))
    for d, B in ((dims(), 0), (dims(dim=100), 0), (dims(dim=100), 1), (dims(dtype="bf16"), 1),
                 (dims(), -1)):
        rc_ws = wan.wan_block_forward(d, B, 16, 16, None, 16, w, 16, 1024, 16, 1 << 30, None)
        msg_ws = wan.last_error()
        rc_na = wan.wan_block_forward_noalloc(d, B, 16, 16, None, 16, w, 16, 1024, None)
        assert rc_na == rc_ws, (B, rc_na, rc_ws)
        assert wan.last_error() == msg_ws


@pytest.mark.parametrize("kw", [dict(dim=384, heads=3, ffn_dim=512), dict(dim=640, heads=5, ffn_dim=512)])
def test_bf16_block_outside_tensor_core_rules_is_refused(lib, kw):
    """A bf16 block whose dim is not a multiple of 256 cannot use the
    tensor-core QKV epilogue; it is refused, never run on other kernels."""
    d = dims(dtype="bf16", **kw)
    w = wan.wan_block_weights(*([4096] * len(wan.WEIGHT_FIELDS)))
    rc = wan.wan_block_forward(d, 1, 16, 16, None, 16, w, 16, 1024, 16, 1 << 40, None)
    assert rc == wan.WAN_EUNSUPPORTED
    assert "256" in wan.last_error()
    assert wan.wan_block_workspace_bytes(d, 1) == 0


def test_release_build_has_no_debug_checks(lib):
    """The product library is the release build; the bounds-checking one is
    libwan_debug.so, loaded only through WAN_LIBRARY."""
    if os.environ.get("WAN_LIBRARY"):
        pytest.skip("WAN_LIBRARY names another build")
    assert wan.wan_debug_bounds() == 0
