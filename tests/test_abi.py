"""The C-ABI library builds, loads and exports every symbol include/ep.h
declares; host-only entry points work without a GPU; a missing library is a
loud error, never a fallback."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    import combine_ep_get_08_b200 as ep
    return ep


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "ep.h")).read()
    names = re.findall(r"EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", text)
    assert len(names) >= 15
    return names


def test_exports_every_declared_symbol(lib):
    so = lib.library()
    missing = [n for n in declared_symbols() if not hasattr(so, n)]
    assert not missing, missing


def test_binding_names_match_abi(lib):
    for n in declared_symbols():
        assert callable(getattr(lib, n, None)), f"binding lacks {n}"


def test_host_only_calls(lib):
    cfg = lib.make_config(4096, 7168, 256, 8, 8, 1)
    assert lib.ep_validate_config(cfg) == 0
    assert lib.ep_capacity_rows(cfg) == 4096 * 8
    assert lib.ep_scales_per_row(cfg) == 56
    assert lib.ep_capacity_rows(lib.make_config(16384, 7168, 256, 64, 8, 128)) == 16384 * 8 + 256 * 127
    bad = [lib.make_config(4, 7168, 256, 7, 8, 1),      # E % R != 0
           lib.make_config(4, 7164, 256, 8, 8, 1),      # H % 8 != 0
           lib.make_config(-1, 256, 8, 2, 2, 1),
           lib.make_config(4, 256, 8, 2, 0, 1),
           lib.make_config(4, 256, 8, 2, 2, 0),
           lib.make_config(4, 256, 8, 16, 2, 1)]        # R > E
    for c in bad:
        assert lib.ep_validate_config(c) == lib.EP_ERR_ARG
    assert lib.ep_validate_config(lib.make_config(4, 256, 2048, 8, 8, 1)) == lib.EP_ERR_UNSUPPORTED
    assert lib.ep_validate_config(lib.make_config(4, 256, 8, 2, 65, 1)) == lib.EP_ERR_UNSUPPORTED
    with pytest.raises(lib.EpError):
        lib.ep_capacity_rows(bad[0])
    assert "invalid" in lib.ep_status_string(lib.EP_ERR_ARG)
    assert lib.ep_launch_count() == 0


def test_missing_library_fails_loudly():
    code = ("import combine_ep_get_08_b200 as ep\n"
            "try:\n    ep.ep_capacity_rows(ep.make_config(1, 8, 1, 1, 1, 1))\n"
            "except RuntimeError as e:\n    print('LOUD', e)\n")
    env = dict(os.environ, EP_B200_LIB="/nonexistent/libep_b200.so")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert "LOUD" in r.stdout and "no CPU fallback" in r.stdout.replace("There is no", "no")


def test_oracle_not_imported_by_product_path():
    pkg = os.path.join(ROOT, "combine_ep_get_08_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f"{f} mentions the oracle"
