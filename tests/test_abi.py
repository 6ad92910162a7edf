"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vsl.h")


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"VSL_API\s+[\w\s\*]+?\b(vsl_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["vsl_logits_local", "vsl_sample", "vsl_sample_workspace_bytes", "vsl_status_string",
              "vsl_device_error", "vsl_version"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    import vocab_sharded_logits_b200 as v
    out = subprocess.run(["nm", "-D", "--defined-only", v.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(vsl_\w+)", out))
    for n in _declared_functions():
        assert n in exported, n
        assert hasattr(v.lib, n)


def test_status_strings_and_version():
    import vocab_sharded_logits_b200 as v
    assert v.status_string(0) == "ok"
    for s in range(1, 7):
        assert v.status_string(s) and v.status_string(s) != "unknown status"
    assert v.status_string(99) == "unknown status"
    assert b"sm_100a" in v.lib.vsl_version()


def test_host_validation_rejects_bad_arguments_without_a_device():
    import vocab_sharded_logits_b200 as v
    L = v.lib
    vp = ctypes.c_void_p
    fake = vp(0x10000)                       # never dereferenced: validation fails first
    arr1 = (vp * 1)(0x10000)
    null_arr = (vp * 1)(0)
    # vsl_logits_local
    assert L.vsl_logits_local(None, arr1, arr1, 4, 64, 1, 512, None) == 1
    assert L.vsl_logits_local(fake, arr1, arr1, 0, 64, 1, 512, None) == 1
    assert L.vsl_logits_local(fake, arr1, arr1, 4, 64, 0, 512, None) == 1
    assert L.vsl_logits_local(fake, arr1, arr1, 4, 64, 17, 512, None) == 3
    assert L.vsl_logits_local(fake, arr1, arr1, 4, 60, 1, 512, None) == 2      # H % 8
    assert L.vsl_logits_local(fake, arr1, arr1, 4, 64, 1, 510, None) == 2      # V_s % 4
    assert L.vsl_logits_local(vp(0x10004), arr1, arr1, 4, 64, 1, 512, None) == 2
    assert L.vsl_logits_local(fake, null_arr, arr1, 4, 64, 1, 512, None) == 1
    # vsl_sample
    args = lambda R=4, S=1, V_s=512, n=5, params=fake, topn=fake, ws=0: (
        arr1, R, S, V_s, params, ctypes.c_uint64(0), n, fake, fake, topn, topn, fake, None, ws, None)
    assert L.vsl_sample(*args(R=0)) == 1
    assert L.vsl_sample(*args(n=-1)) == 1
    assert L.vsl_sample(*args(n=21)) == 3
    assert L.vsl_sample(*args(S=1, V_s=4, n=5)) == 1          # n > V
    assert L.vsl_sample(*args(params=None)) == 1
    assert L.vsl_sample(*args(topn=None)) == 1
    assert L.vsl_sample(*args(V_s=514)) == 2
    assert L.vsl_sample(*args(S=17)) == 3
    assert L.vsl_sample(*args(V_s=1 << 20, S=1)) == 3         # beyond the largest vocabulary
    assert L.vsl_sample_workspace_bytes(2048, 8, 18992, 20) == 0
    # vsl_verify_drafts
    L.vsl_verify_drafts.argtypes = [vp] * 3 + [ctypes.c_int32] * 2 + [vp] * 4
    assert L.vsl_verify_drafts(None, None, fake, 4, 3, fake, None, fake, None) == 1     # no tokens
    assert L.vsl_verify_drafts(fake, None, fake, 0, 3, fake, None, fake, None) == 1     # no requests
    assert L.vsl_verify_drafts(fake, None, fake, 4, -1, fake, None, fake, None) == 1    # negative spec
    assert L.vsl_verify_drafts(fake, None, fake, 4, 65, fake, None, fake, None) == 1    # spec > VSL_MAX_SPEC
    assert L.vsl_verify_drafts(fake, None, None, 4, 3, fake, None, fake, None) == 1     # drafts missing
    assert L.vsl_verify_drafts(fake, fake, fake, 4, 3, fake, None, fake, None) == 1     # one logprob pointer
    # vsl_sample_ex: the same checks, plus the optional outputs' alignment
    ex = lambda extras, **kw: L.vsl_sample_ex(*args(**kw)[:-1], extras, None)
    assert ex(None, R=0) == 1
    assert ex(ctypes.byref(v._Extras(0x10004)), V_s=512) == 2         # kept_theta not 8-byte aligned
    assert ex(ctypes.byref(v._Extras(0x10008)), V_s=1 << 20) == 3     # aligned: the size check follows
    assert ex(ctypes.byref(v._Extras(0, 0x10000)), V_s=512) == 1       # processed without kept_theta
    assert ex(ctypes.byref(v._Extras(0x10008, 0x10000)), V_s=512) == 1 # processed top-n missing (n = 5)
    assert ex(ctypes.byref(v._Extras(0, 0, 0x10000)), V_s=512) == 1    # processed top-n without the token's
    assert ex(ctypes.byref(v._Extras(0, 0, 0, 0, 0x10010)), V_s=512) == 2  # tile statistics not 32-byte aligned
    # tile statistics: sizes, and the checks of both producers
    assert L.vsl_tile_stats_floats(4, 2, 300) == 4 * 2 * 3 * 8
    assert L.vsl_tile_stats_floats(0, 2, 300) == 0
    assert L.vsl_tile_stats(None, 4, 1, 512, fake, None) == 1
    assert L.vsl_tile_stats(arr1, 4, 1, 512, None, None) == 1
    assert L.vsl_tile_stats(arr1, 0, 1, 512, fake, None) == 1
    assert L.vsl_tile_stats(arr1, 4, 17, 512, fake, None) == 3
    assert L.vsl_tile_stats(arr1, 4, 1, 510, fake, None) == 2                # V_s % 4
    assert L.vsl_tile_stats(arr1, 4, 1, 512, vp(0x10010), None) == 2         # records not 32-byte aligned
    assert L.vsl_tile_stats((vp * 1)(0x10004), 4, 1, 512, fake, None) == 2   # slice not 16-byte aligned
    assert L.vsl_logits_local_ex(fake, arr1, arr1, 4, 64, 1, 512, vp(0x10010), None) == 2
    assert L.vsl_logits_local_ex(fake, arr1, arr1, 0, 64, 1, 512, fake, None) == 1


def test_binding_has_no_cpu_fallback(monkeypatch, tmp_path):
    """The binding raises at import when the library is absent."""
    import importlib.util
    import shutil
    pkg = os.path.join(ROOT, "vocab_sharded_logits_b200")
    dst = tmp_path / "vocab_sharded_logits_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    spec = importlib.util.spec_from_file_location("vsl_nolib", dst / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_sample_launches_rejects_bad_sizes_on_the_host():
    import vocab_sharded_logits_b200 as v
    lib = v.lib
    assert lib.vsl_sample_launches(0, 4, 37984) == -1
    assert lib.vsl_sample_launches(64, 0, 37984) == -1
    assert lib.vsl_sample_launches(64, 17, 37984) == -1
    assert lib.vsl_sample_launches(64, 4, 37983) == -1
