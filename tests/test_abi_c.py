"""The C ABI from a plain C11 program: include/tile3d.h compiles as C with warnings as errors, the
program links against libtile3d.so, and its host-side calls (geometry, validation failures) agree
with the oracle without a GPU."""
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import tiling

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "block_sparse_video_tile3d_b200")


@pytest.fixture(scope="module")
def abi_check():
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    if not os.path.exists(os.path.join(LIBDIR, "libtile3d.so")):
        pytest.skip("libtile3d.so not built")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "abi_check")
        subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_check.c"),
                        "-L", LIBDIR, "-ltile3d", "-Wl,-rpath," + LIBDIR, "-o", exe],
                       check=True, capture_output=True, text=True)
        yield exe


def _run(exe, *args):
    out = subprocess.run([exe, *map(str, args)], check=True, capture_output=True, text=True).stdout
    return dict(line.split(" ", 1) for line in out.strip().splitlines())


@pytest.mark.parametrize("grid", [(4, 8, 8), (21, 30, 52), (3, 5, 7), (1, 1, 1), (16, 32, 56)])
def test_c_program_geometry_matches_oracle(abi_check, grid):
    r = _run(abi_check, 1, *grid, 2, 64)
    want = tiling.variable_block_sizes(*grid)
    assert int(r["nT"].split()[0]) == len(want)
    assert r["nT"].split()[2] == str(64 * len(want))
    np.testing.assert_array_equal(np.array(r["vc"].split(), dtype=np.int64), want)
    assert r["version"].strip()


def test_c_program_validation_failures(abi_check):
    r = _run(abi_check, 1, 4, 8, 8, 2, 64)
    assert r["scatter_null"] == "1"  # T3D_ERR_INVALID
    assert r["topk_k0"] == "1"
    assert r["ws_null_geom"] == "0"


@pytest.mark.parametrize("args,status", [((1, 4, 8, 8, 2, 96), "2"),   # D not in {64, 128}
                                         ((0, 4, 8, 8, 2, 64), "1"),   # empty batch
                                         ((1, 4, 8, 0, 2, 64), "1")])  # empty grid
def test_c_program_geometry_rejections(abi_check, args, status):
    r = _run(abi_check, *args)
    assert r["geometry_status"].split()[0] == status
    assert "vc" not in r
