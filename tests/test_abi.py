"""The C-ABI library: it loads, exports every symbol its header declares, and
its host-side validation and error paths behave without a GPU."""
import ctypes
import os
import re
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def _declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b([a-z_][a-z0-9_]*)\s*\(", text):
            name = m.group(1)
            if name.startswith(("spectre_", "dct_mix_")) and name not in names:
                names.append(name)
    return names


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for required in ["spectre_mix_create", "spectre_mix_run", "spectre_mix_run_debug",
                     "spectre_mix_run_host", "spectre_mix_destroy", "spectre_mix_error_string",
                     "spectre_mix_workspace_bytes", "spectre_mix_plan_info", "dct_mix_create",
                     "dct_mix_run", "dct_mix_run_debug", "dct_mix_run_host", "dct_mix_destroy"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    from sub_quadratic_attention_b200 import binding

    lib = ctypes.CDLL(binding.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in binding.SIGNATURES, name


def test_error_strings_are_distinct():
    from sub_quadratic_attention_b200 import binding as b

    codes = [b.SPECTRE_OK, b.SPECTRE_ERR_ARG, b.SPECTRE_ERR_UNSUPPORTED_L, b.SPECTRE_ERR_ALIGN,
             b.SPECTRE_ERR_CUDA, b.SPECTRE_ERR_NOMEM, b.SPECTRE_ERR_DEVICE]
    texts = [b.spectre_mix_error_string(c) for c in codes]
    assert len(set(texts)) == len(texts)
    assert "unknown" in b.spectre_mix_error_string(12345)


@pytest.mark.parametrize("args,code", [
    ((0, 256, 1, 16, 129, 0), "SPECTRE_ERR_ARG"),        # B < 1
    ((1, 256, 0, 16, 129, 0), "SPECTRE_ERR_ARG"),        # H < 1
    ((1, 256, 1, 0, 129, 0), "SPECTRE_ERR_ARG"),         # D < 1
    ((1, 256, 1, 16, 130, 0), "SPECTRE_ERR_ARG"),        # F > L/2 + 1
    ((1, 256, 1, 16, 0, 0), "SPECTRE_ERR_ARG"),          # F < 1
    ((1, 256, 1, 16, 129, 7), "SPECTRE_ERR_ARG"),        # dtype
    ((1, 100, 1, 16, 51, 0), "SPECTRE_ERR_UNSUPPORTED_L"),
    ((1, 4, 1, 16, 3, 0), "SPECTRE_ERR_UNSUPPORTED_L"),
    ((1, 1 << 21, 1, 16, 5, 0), "SPECTRE_ERR_UNSUPPORTED_L"),
    ((1, 5 * 1024, 1, 16, 5, 0), "SPECTRE_ERR_UNSUPPORTED_L"),
    ((1, 1 << 20, 8, 512, 5, 1), "SPECTRE_ERR_ARG"),     # C too wide for the R = 64 row pass
    ((1, 1 << 20, 1, 865, 5, 1), "SPECTRE_ERR_ARG"),     # C = 865 > 864, the R = 64 limit
    ((1, 1 << 18, 1, 3617, 5, 1), "SPECTRE_ERR_ARG"),    # C = 3617 > 3616, the R = 16 limit
    ((65536, 256, 1, 16, 129, 0), "SPECTRE_ERR_ARG"),    # B above 65535
    ((1, 256, 1024, 1025, 129, 0), "SPECTRE_ERR_ARG"),   # H * D above 2^20
])
def test_create_validates_before_touching_the_device(args, code):
    from sub_quadratic_attention_b200 import binding as b

    st, h = b.spectre_mix_create_status(*args)
    assert st == getattr(b, code)
    assert h is None


def test_create_rejects_bad_eps():
    from sub_quadratic_attention_b200 import binding as b

    for eps in (0.0, -1.0, float("nan"), float("inf")):
        st, h = b.spectre_mix_create_status(1, 256, 1, 16, 129, 0, eps)
        assert st == b.SPECTRE_ERR_ARG and h is None


def test_null_handle_paths():
    from sub_quadratic_attention_b200 import binding as b

    assert b._lib.spectre_mix_set_option(None, b.SPECTRE_OPT_TENSOR_CORES, 1) == b.SPECTRE_ERR_ARG
    assert b._lib.spectre_mix_slice_pass(None) == b.SPECTRE_ERR_ARG
    assert b._lib.spectre_mix_set_option(None, b.SPECTRE_OPT_NORM, 1) == b.SPECTRE_ERR_ARG
    assert b._lib.spectre_mix_device_status(None, None) == b.SPECTRE_ERR_ARG
    b.spectre_mix_destroy(None)                      # NULL-safe
    assert b.spectre_mix_workspace_bytes(None) == 0
    with pytest.raises(b.SpectreMixError):
        b.spectre_mix_plan_info(None)
    assert b.spectre_mix_run_status(None, *([0] * 8), stream=0) == b.SPECTRE_ERR_ARG


def _run_child(code: str, env_extra: dict) -> str:
    env = dict(os.environ)
    env.update(env_extra)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         timeout=120)
    assert out.returncode == 0, out.stderr
    return out.stdout.strip()


def test_allocation_fault_injection_is_reported():
    code = ("from sub_quadratic_attention_b200 import binding as b\n"
            "st, h = b.spectre_mix_create_status(1, 256, 1, 16, 129, 0)\n"
            "print(st, h)")
    assert _run_child(code, {"SPECTRE_MIX_FAULT": "alloc"}) == "-5 None"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_create_without_a_device_reports_device_error():
    from sub_quadratic_attention_b200 import binding as b

    st, h = b.spectre_mix_create_status(1, 256, 1, 16, 129, 0)
    assert st == b.SPECTRE_ERR_DEVICE and h is None


@pytest.mark.parametrize("args,code", [
    ((32, 0), "SPECTRE_ERR_UNSUPPORTED_L"),        # d below 64
    ((96, 0), "SPECTRE_ERR_UNSUPPORTED_L"),        # not a power of two
    ((2048, 1), "SPECTRE_ERR_UNSUPPORTED_L"),      # above 1024
    ((256, 2), "SPECTRE_ERR_ARG"),                 # dtype
])
def test_dct_create_validates_before_touching_the_device(args, code):
    from sub_quadratic_attention_b200 import binding as b

    st, h = b.dct_mix_create_status(*args)
    assert st == getattr(b, code) and h is None
    for eps in (0.0, float("nan")):
        st, h = b.dct_mix_create_status(256, 0, eps)
        assert st == b.SPECTRE_ERR_ARG and h is None


def test_dct_null_handle_paths():
    from sub_quadratic_attention_b200 import binding as b

    assert b._lib.dct_mix_destroy(None) == b.SPECTRE_OK
    assert b._lib.dct_mix_run(None, 4, *([None] * 4), 0.5, *([None] * 4)) == b.SPECTRE_ERR_ARG
    assert b._lib.dct_mix_run_host(None, 4, *([None] * 4), 0.5, *([None] * 4)) == b.SPECTRE_ERR_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_dct_create_without_a_device_reports_device_error():
    from sub_quadratic_attention_b200 import binding as b

    st, h = b.dct_mix_create_status(256, 1)
    assert st == b.SPECTRE_ERR_DEVICE and h is None
