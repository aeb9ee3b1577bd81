"""The C-ABI library: it loads without a GPU, exports every entry point the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from mixture_experts_layer_64_b200 import build, lmoe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def L():
    build.build_library()
    return lmoe.lib()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(lmoe_\w+)\s*\(", text, re.M):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 18
    for n in sorted(names):
        assert hasattr(L, n), f"{n} declared but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\b(lmoe_\w+)\b", out))
    assert names <= exported
    assert set(lmoe.EXPORTS) <= names


def test_library_has_no_driver_link_dependency():
    # the .so loads on a machine without libcuda: it resolves the driver at run time
    out = subprocess.run(["ldd", build.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out
    assert "torch" not in out


def test_status_strings_and_stage_names(L):
    for s in range(8):
        assert lmoe.status_string(s)
    assert lmoe.status_string(0) == "ok"
    names = [lmoe.stage_name(i) for i in range(9)]
    assert names == ["router", "topk", "group", "down_proj", "shared_fc1", "expert_fc1",
                     "expert_fc2", "combine", "up_proj"]
    assert lmoe.stage_name(9) == ""


@pytest.mark.parametrize("args", [
    (0, 64, 16, 4, 128, 0, 0, 0, 0),          # d = 0
    (256, 64, 16, 17, 128, 0, 0, 0, 0),       # k > N
    (256, 64, 16, 0, 128, 0, 0, 0, 0),        # k = 0
    (256, 64, 16, 4, 128, 7, 0, 0, 0),        # unknown act
    (256, 64, 16, 4, 128, 0, 0, 5, 0),        # unknown dtype
    (256, 64, 16, 4, 128, 0, -1, 0, 0),       # negative shared width
    (256, 64, 16, 4, 128, 0, 0, 0, 1),        # skip flag with l != d
    (256, 256, 16, 4, 128, 0, 0, 0, 0x8 | 0x10),  # contradictory forcing flags
    (256, 256, 16, 4, 128, 0, 0, 0, 0x20000),  # unknown flag
])
def test_create_rejects_bad_arguments(L, args):
    h = ctypes.c_void_p(123)
    st = L.lmoe_create(*args, ctypes.byref(h))
    assert st == lmoe.ERR_INVALID_ARG
    assert not h.value


def test_create_reports_unsupported_limits(L):
    h = ctypes.c_void_p()
    assert L.lmoe_create(64, 64, 2048, 4, 64, 0, 0, 1, 0, ctypes.byref(h)) == lmoe.ERR_UNSUPPORTED
    assert L.lmoe_create(64, 64, 64, 33, 64, 0, 0, 1, 0, ctypes.byref(h)) == lmoe.ERR_UNSUPPORTED
    assert L.lmoe_create(64, 64, 16, 4, 64, 0, 0, 1, 0, None) == lmoe.ERR_INVALID_ARG


def test_null_handle_calls_fail_cleanly(L):
    I = ctypes.c_int
    assert L.lmoe_set_weights(None, *([None] * 8)) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_reserve(None, 16) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_forward(None, None, None, 4, None) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_forward_host(None, None, None, 4, None) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_route_only(None, None, 4, None, None, None, None, None) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_router_logits(None, None, None, 4, None) == lmoe.ERR_INVALID_ARG
    n = ctypes.c_size_t()
    assert L.lmoe_stage_bytes(None, 0, 4, ctypes.byref(n)) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_debug_dump(None, 0, None, 0, None) == lmoe.ERR_INVALID_ARG
    w = I()
    assert L.lmoe_last_error(None, ctypes.byref(w)) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_profile_begin(None, 4) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_profile_end(None, None, 0, ctypes.byref(w), ctypes.byref(w)) == lmoe.ERR_INVALID_ARG
    assert L.lmoe_last_launch_count(None) == 0
    assert L.lmoe_last_expert_path(None) == -1
    assert L.lmoe_error_detail(None) == b""
    L.lmoe_destroy(None)


def test_binding_refuses_to_run_without_a_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(RuntimeError):
        lmoe.LatentMoELayer(256, 64, 16, 4, 128, act="silu", dtype="f32")
