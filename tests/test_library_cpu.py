"""The C-ABI library without a GPU: it loads, exports every declared entry
point, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as fh:
                text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", text, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from intra_expert_activation_router_b200 import build
    build.build()
    import intra_expert_activation_router_b200 as m
    return m


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("moe_sparse_create", "moe_sparse_forward", "moe_dense_forward", "moe_sparse_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(so, n)]
    assert not missing, missing
    assert set(declared_functions()) <= set(lib.EXPORTED)


def test_strerror(lib):
    assert lib.moe_strerror(0) == "success"
    for c in (lib.MOE_EINVAL, lib.MOE_ENOMEM, lib.MOE_ECUDA, lib.MOE_EALIGN, lib.MOE_EHANDLE,
              lib.MOE_EDEVICE, lib.MOE_ENOTSUP):
        assert lib.moe_strerror(c) not in ("success", "unknown error code")
    assert lib.moe_strerror(12345) == "unknown error code"


def _weights(lib, **over):
    base = dict(w_router=0x10000, w_gate=0x20000, w_up=0x30000, w_down=0x40000)
    base.update(over)
    return lib._binding.moe_weights(*[base.get(n) for n, _ in lib._binding.moe_weights._fields_])


def _create(lib, w, E=8, k=2, d=256, f=512, S=0, maxT=16):
    h = ctypes.c_void_p()
    return lib.raw_call("moe_sparse_create", ctypes.byref(w), E, k, d, f, S, maxT, ctypes.byref(h))


@pytest.mark.parametrize("kw,code", [
    (dict(E=0), -1), (dict(E=2000), -1), (dict(k=0), -1), (dict(k=9), -1),
    (dict(d=260 - 1), -1), (dict(d=0), -1), (dict(d=4104), -1), (dict(f=48), -1), (dict(f=65536 + 32), -1),
    (dict(S=-1), -1), (dict(S=9), -1), (dict(maxT=-3), -1), (dict(maxT=70000), -1),
    (dict(S=1), -1),          # shared count without shared weights
])
def test_create_rejects_bad_sizes(lib, kw, code):
    assert _create(lib, _weights(lib), **kw) == code


def test_create_rejects_null_and_misaligned(lib):
    h = ctypes.c_void_p()
    assert lib.raw_call("moe_sparse_create", None, 8, 2, 256, 512, 0, 16, ctypes.byref(h)) == lib.MOE_EINVAL
    assert lib.raw_call("moe_sparse_create", ctypes.byref(_weights(lib)), 8, 2, 256, 512, 0, 16, None) == lib.MOE_EINVAL
    assert _create(lib, _weights(lib, w_gate=None)) == lib.MOE_EINVAL
    assert _create(lib, _weights(lib, w_up=0x30008)) == lib.MOE_EALIGN
    assert _create(lib, _weights(lib, ws_gate=0x50000)) == lib.MOE_EINVAL   # shared weights with S=0


def test_calls_on_null_or_foreign_handle(lib):
    for name, args in (("moe_sparse_forward", (0x1000, 1, ctypes.c_float(1.0), 0x2000, None)),
                       ("moe_dense_forward", (0x1000, 1, 0x2000, None)),
                       ("moe_set_path", (1,)), ("moe_set_t_star", (4,))):
        for h in (None, 0xdead0):
            assert lib.raw_call(name, h, *args) == lib.MOE_EHANDLE
    lib.moe_sparse_destroy(None)       # ignored
    lib.moe_sparse_destroy(0xdead0)    # not a live handle: ignored


def test_create_without_gpu_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _create(lib, _weights(lib)) == lib.MOE_ECUDA


def test_layer_output_check_on_host(lib):
    """The layer class checks `out` before any launch (CPU tensors stand in)."""
    import torch
    x = torch.zeros(4, 8, dtype=torch.bfloat16)
    good = torch.empty_like(x)
    assert lib.MoESparseLayer._out_like(x, good) is good
    assert lib.MoESparseLayer._out_like(x, None).shape == x.shape
    for bad in (torch.empty(3, 8, dtype=torch.bfloat16), torch.empty(4, 8, dtype=torch.float32),
                torch.empty(8, 4, dtype=torch.bfloat16).t()):
        with pytest.raises(ValueError):
            lib.MoESparseLayer._out_like(x, bad)
