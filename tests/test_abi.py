"""The C-ABI library builds for sm_100a, loads, and exports every entry point
include/mla.h declares (no compute calls: this runs without a GPU)."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for f in ("mla_cache_append", "mla_absorb_q", "mla_decode", "mla_out_proj", "mla_workspace_size",
              "mla_get_device_error", "mla_status_string"):
        assert f in names


def test_library_exports_every_declared_symbol():
    from mla_latent_kv_33_b200 import build
    lib = ctypes.CDLL(build.build())
    missing = [f for f in declared_functions() if not hasattr(lib, f)]
    assert not missing, missing
    lib.mla_status_string.restype = ctypes.c_char_p
    assert lib.mla_status_string(0) == b"MLA_OK"
    assert lib.mla_status_string(6) == b"MLA_ERR_DEVICE_DATA"


def test_launch_overlap_switch_round_trips():
    from mla_latent_kv_33_b200 import build
    lib = ctypes.CDLL(build.build())
    assert lib.mla_get_launch_overlap() == 0  # off by default
    assert lib.mla_set_launch_overlap(1) == 0
    assert lib.mla_get_launch_overlap() == 1
    assert lib.mla_set_launch_overlap(0) == 0
    assert lib.mla_get_launch_overlap() == 0
