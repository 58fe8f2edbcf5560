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
    # peer / IPC calls reject null arguments on the host, before any CUDA call
    c = lib.library()
    assert c.ep_dispatch_peer(None, None, None, None, None) == lib.EP_ERR_ARG
    assert c.ep_combine_peer(None, None, None, None, None, None) == lib.EP_ERR_ARG
    assert c.ep_ipc_get_handle(None, None, None) == lib.EP_ERR_ARG
    assert c.ep_ipc_open_handle(None, None) == lib.EP_ERR_ARG
    assert c.ep_ipc_close_handle(None) == lib.EP_ERR_ARG
    with pytest.raises(ValueError):
        lib.ep_ipc_open_handle(b"short")
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


C_PROGRAM = r"""
#include <stdio.h>
#include "ep.h"

int main(void) {
    ep_config c = {4096, 7168, 256, 8, 8, 128};
    if (ep_validate_config(&c) != EP_OK) return 1;
    if (ep_capacity_rows(&c) != 4096LL * 8 + 256LL * 127) return 2;
    if (ep_scales_per_row(&c) != 56) return 3;
    if (ep_scale_buffer_floats(&c, EP_SCALES_COL_MAJOR_TMA) != 56LL * ((ep_capacity_rows(&c) + 3) / 4 * 4)) return 4;
    if (ep_ll_capacity_rows(&c, 4096) != 256LL * 4096) return 5;
    if (ep_ll_capacity_rows(&c, 100) != EP_ERR_ARG) return 6;   /* fewer slots than tokens */
    c.num_ranks = 7;
    if (ep_validate_config(&c) != EP_ERR_ARG) return 7;
    printf("ok %s\n", ep_status_string(EP_ERR_STATE));
    return 0;
}
"""


def test_header_is_c99_and_links(lib, tmp_path):
    """A plain C99 program compiles against include/ep.h with warnings as
    errors, links against libep_b200.so and runs its host-only calls."""
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:libep_b200.so", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.startswith("ok ")
