"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/isd.h declares, sizes workspaces, and rejects bad arguments on
the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def isd():
    from speculative_verification_isd_b200 import build as B
    B.build()
    from speculative_verification_isd_b200 import isd as lib
    return lib


def declared_functions():
    text = open(os.path.join(ROOT, "include", "isd.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(isd_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(isd):
    names = declared_functions()
    assert "isd_step" in names and "isd_accept" in names
    lib = ctypes.CDLL(isd.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(isd.EXPORTED) == set(names)


def test_status_strings(isd):
    lib = isd.library()
    assert lib.isd_status_string(0) == b"ISD_OK"
    assert lib.isd_status_string(-3) == b"ISD_ERR_WORKSPACE"
    assert lib.isd_status_string(7) == b"ISD_ERR_UNKNOWN"


def test_workspace_sizes(isd):
    from speculative_verification_isd_b200 import inputs as I
    for name, cfg in I.CONFIGS.items():
        d = isd.make_dims(cfg.B, cfg.N, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, cfg.page_size, 100,
                          cfg.max_pages_per_req(), cfg.lora_rank)
        n = isd.workspace_bytes(d)
        assert n > 0 and n % 256 == 0, name
        assert n >= cfg.M * cfg.H * 2
    bad = isd.make_dims(2, 2, 4, 3, 64, 10, 16, 10, 4)   # Hq % Hkv != 0
    assert isd.workspace_bytes(bad) == 0
    bad = isd.make_dims(2, 0, 4, 1, 64, 10, 16, 10, 4)   # N = 0
    assert isd.workspace_bytes(bad) == 0


def test_host_validation_rejects_before_launch(isd):
    lib = isd.library()
    d = isd.make_dims(2, 2, 4, 1, 64, 512, 16, 10, 4)
    need = isd.workspace_bytes(d)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    p = [fake] * 10
    # missing workspace
    st = lib.isd_attention(ctypes.byref(d), *p, 0, None, None)
    assert st == isd.ISD_ERR_WORKSPACE
    # misaligned workspace
    st = lib.isd_attention(ctypes.byref(d), *p[:9], ctypes.c_void_p((1 << 20) + 8), need, None,
                           None)
    assert st == isd.ISD_ERR_WORKSPACE
    # null tensor pointer
    st = lib.isd_attention(ctypes.byref(d), None, *p[1:], need, None, None)
    assert st == isd.ISD_ERR_INVALID_ARG
    # unsupported head dim
    d2 = isd.make_dims(2, 2, 4, 1, 96, 512, 16, 10, 4)
    st = lib.isd_attention(ctypes.byref(d2), *p, isd.workspace_bytes(d2), None, None)
    assert st == isd.ISD_ERR_UNSUPPORTED_SHAPE
    # hidden size not a multiple of 64 for the tensor-core LM head
    d3 = isd.make_dims(2, 2, 1, 1, 32, 512, 16, 10, 4)
    st = lib.isd_lm_head(ctypes.byref(d3), fake, fake, None, None, fake, fake, fake,
                         isd.workspace_bytes(d3), None, None)
    assert st == isd.ISD_ERR_UNSUPPORTED_SHAPE
    # LoRA pointers without a rank
    st = lib.isd_lm_head(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, need, None,
                         None)
    assert st == isd.ISD_ERR_INVALID_ARG
    # bad proposal mode
    d4 = isd.make_dims(2, 2, 4, 1, 64, 512, 16, 10, 4, proposal_mode=5)
    assert isd.workspace_bytes(d4) == 0
    assert b"invalid" in lib.isd_last_error() or b"unsupported" in lib.isd_last_error()


def test_binding_checks_tensors_on_host(isd):
    import torch
    d = isd.make_dims(2, 2, 4, 1, 64, 512, 16, 10, 4)
    with pytest.raises(ValueError):
        isd._ptr(torch.zeros(4), torch.float32, 4, "cpu tensor")


def test_binding_prototypes_match_header(isd):
    """Every ctypes prototype has the header's parameter count and kinds."""
    text = open(os.path.join(ROOT, "include", "isd.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lib = isd.library()
    for name in declared_functions():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)\s*;", text, flags=re.S)
        assert m, name
        params = [p.strip() for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        argtypes = getattr(lib, name).argtypes
        assert len(argtypes) == len(params), (name, len(argtypes), len(params))
        for p, a in zip(params, argtypes):
            if "*" in p:
                assert a in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(a, "_type_"), (name, p)
            elif p.startswith("size_t"):
                assert a is ctypes.c_size_t, (name, p)
            elif p.startswith("float"):
                assert a is ctypes.c_float, (name, p)
            else:
                assert a is ctypes.c_int32, (name, p)


def test_sdar_host_validation(isd):
    """The SDAR-style calls reject bad dims and pointers on the host."""
    lib = isd.library()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    d = isd.make_dims(2, 4, 4, 1, 128, 512, 16, 10, 4)
    need = isd.workspace_bytes(d)
    p16 = [fake] * 16
    ok = lambda dd, tau, args: lib.isd_sdar_step(ctypes.byref(dd), tau, 1, *args, fake, need,
                                                 None, None)
    assert ok(d, float("nan"), p16) == isd.ISD_ERR_INVALID_ARG
    assert ok(d, 0.5, [None] + p16[1:]) == isd.ISD_ERR_INVALID_ARG        # q
    assert ok(d, 0.5, p16[:7] + [None] + p16[8:]) == isd.ISD_ERR_INVALID_ARG  # W
    d_lora = isd.make_dims(2, 4, 4, 1, 128, 512, 16, 10, 4, lora_rank=32)
    st = lib.isd_sdar_step(ctypes.byref(d_lora), 0.5, 1, *p16, fake,
                           isd.workspace_bytes(d_lora), None, None)
    assert st == isd.ISD_ERR_UNSUPPORTED_SHAPE
    d_wide = isd.make_dims(2, 17, 4, 1, 128, 512, 16, 10, 8)
    st = lib.isd_sdar_unmask(ctypes.byref(d_wide), 0.5, 1, *[fake] * 7, fake,
                             isd.workspace_bytes(d_wide), None, None)
    assert st == isd.ISD_ERR_UNSUPPORTED_SHAPE
    st = lib.isd_sdar_unmask(ctypes.byref(d), 0.5, 1, None, *[fake] * 6, fake, need, None, None)
    assert st == isd.ISD_ERR_INVALID_ARG
    # workspace too small
    st = lib.isd_sdar_unmask(ctypes.byref(d), 0.5, 1, *[fake] * 7, fake, 256, None, None)
    assert st == isd.ISD_ERR_WORKSPACE
    st = lib.isd_sdar_loop(ctypes.byref(d), 0.5, 1, 4, None, fake, need, None, None)
    assert st == isd.ISD_ERR_INVALID_ARG


def test_full_depth_host_validation(isd):
    """isd_layers / isd_embed_block reject bad sizes and pointers on the host."""
    lib = isd.library()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    d = isd.make_dims(2, 4, 4, 2, 64, 500, 16, 10, 4)
    assert isd.layers_workspace_bytes(d, 96) > isd.workspace_bytes(d)
    assert isd.layers_workspace_bytes(d, 100) == 0          # intermediate not a multiple of 8
    assert isd.layers_workspace_bytes(isd.make_dims(2, 0, 4, 2, 64, 500, 16, 10, 4), 96) == 0
    need = isd.layers_workspace_bytes(d, 96)
    arr = (isd.Layer * 1)()
    for n in isd.LAYER_FIELDS:
        setattr(arr[0], n, 1 << 20)
    call = lambda **kw: lib.isd_layers(
        ctypes.byref(kw.get("d", d)), kw.get("n", 1), kw.get("inter", 96), 1e-6,
        kw.get("layers", arr), kw.get("rope", fake), kw.get("rope_n", 64), None,
        kw.get("x", fake), None, fake, fake, fake, kw.get("ws", fake), kw.get("ws_bytes", need),
        None, None)
    assert call(inter=100) == isd.ISD_ERR_INVALID_ARG
    assert call(ws_bytes=need - 256) == isd.ISD_ERR_WORKSPACE
    assert call(x=None) == isd.ISD_ERR_INVALID_ARG
    assert call(rope=None) == isd.ISD_ERR_INVALID_ARG
    assert call(rope_n=0) == isd.ISD_ERR_INVALID_ARG
    assert call(n=-1) == isd.ISD_ERR_INVALID_ARG
    assert call(layers=None) == isd.ISD_ERR_INVALID_ARG
    bad = (isd.Layer * 1)()
    for n in isd.LAYER_FIELDS:
        setattr(bad[0], n, 1 << 20)
    bad[0].w_down = None
    assert call(layers=bad) == isd.ISD_ERR_INVALID_ARG
    d96 = isd.make_dims(2, 4, 4, 2, 96, 500, 16, 10, 4)     # head dim the attention lacks
    assert call(d=d96, ws_bytes=isd.layers_workspace_bytes(d96, 96)) == isd.ISD_ERR_UNSUPPORTED_SHAPE
    assert lib.isd_embed_block(ctypes.byref(d), None, fake, fake, fake, None, None) == \
        isd.ISD_ERR_INVALID_ARG
