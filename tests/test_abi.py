"""The C-ABI library: builds for sm_100a, loads, exports every function that
include/moe.h declares, and its host-side argument checks behave (no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    from int4_routed_expert_softmax_b200 import build
    build.build()
    import int4_routed_expert_softmax_b200 as moe
    return moe.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\**\s*((?:moe|expert_cache)_\w+)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("moe_router_topk", "moe_bucket", "moe_layer_forward", "moe_quant_q8_0",
                 "moe_workspace_bytes", "moe_expert_bytes"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        getattr(lib, n)


def test_dims_and_sizes(lib):
    import int4_routed_expert_softmax_b200 as moe
    d = moe.dims(6144, 2048, 256, 8)
    assert moe.moe_check_dims(d) == 0
    assert moe.moe_expert_bytes(d) == 20_054_016
    assert moe.moe_expert_bytes(moe.dims(256, 128, 16, 2)) == 52_224
    sizes = [moe.moe_workspace_bytes(d, T) for T in (0, 1, 4, 16, 2048)]
    assert all(s % 256 == 0 and s > 0 for s in sizes)
    assert sizes == sorted(sizes)
    for bad in [(200, 128, 16, 2), (256, 100, 16, 2), (256, 128, 16, 17), (256, 128, 0, 1),
                (256, 128, 16, 0), (256, 128, 2000, 2), (256, 128, 64, 33), (16384, 128, 4, 2)]:
        assert moe.moe_check_dims(moe.dims(*bad)) == -2, bad
        assert moe.moe_expert_bytes(moe.dims(*bad)) == 0
    assert moe.moe_workspace_bytes(d, -1) == 0
    for code in range(-9, 1):
        assert moe.status_string(code) != "unknown status"


def test_host_side_argument_errors(lib):
    """Rejected on the host before any CUDA call is made."""
    import int4_routed_expert_softmax_b200 as moe
    d = moe.dims(256, 128, 16, 2)
    P = ctypes.c_void_p
    fake = P(4096)
    L = lib
    assert L.moe_layer_forward(ctypes.byref(d), 1, None, fake, fake, fake, fake, 1 << 20, None, 0, None) == -1
    assert L.moe_layer_forward(ctypes.byref(d), 1, fake, fake, fake, fake, fake, 1 << 20, None, 7, None) == -1
    assert L.moe_layer_forward(ctypes.byref(d), -1, fake, fake, fake, fake, fake, 1 << 20, None, 0, None) == -1
    assert L.moe_layer_forward(ctypes.byref(d), 1, fake, fake, fake, fake, P(4096 + 64), 1 << 20, None, 0, None) == -4
    assert L.moe_layer_forward(ctypes.byref(d), 1, fake, fake, fake, fake, fake, 16, None, 0, None) == -4
    bad = moe.dims(250, 128, 16, 2)
    assert L.moe_layer_forward(ctypes.byref(bad), 1, fake, fake, fake, fake, fake, 1 << 20, None, 0, None) == -2
    assert L.moe_layer_forward(ctypes.byref(d), 0, None, None, None, None, None, 0, None, 0, None) == 0
    assert L.moe_quant_q8_0(fake, 1, 33, fake, fake, None) == -2
    assert L.moe_quant_q8_0(None, 1, 32, fake, fake, None) == -1
    assert L.moe_router_topk(ctypes.byref(d), 1, P(4100), fake, fake, fake, fake, None, None) == -1
    assert L.moe_bucket(ctypes.byref(d), 1, fake, None, fake, fake, fake, fake, None) == -1


def test_oracle_is_separate_from_the_product():
    """The product package never imports the oracle (test infrastructure)."""
    pkg = os.path.join(ROOT, "int4_routed_expert_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in txt and "oracle.h" not in txt and "liboracle" not in txt, f


def test_header_is_c99_and_host_calls_work_from_c(lib, tmp_path):
    """The boundary is a C ABI: a C99 program (-Wall -Wextra -Werror -pedantic)
    includes moe.h, links libmoe.so and runs the host-only calls (status names,
    shape checks, sizes, the route-usage record) without a GPU."""
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
  moe_dims d = {6144, 2048, 256, 8};
  uint64_t c[2 * 4] = {1, 2, 3, 4, 5, 6, 7, (uint64_t)1 << 40}, r[2 * 4];
  if (moe_check_dims(&d) != MOE_OK) return 1;
  if (moe_expert_bytes(&d) != (size_t)20054016) return 2;
  if (strcmp(moe_status_string(MOE_ERR_IO), "unknown status") == 0) return 3;
  if (moe_usage_save(USAGE_PATH, 2, 4, c) != MOE_OK) return 4;
  memset(r, 0, sizeof r);
  if (moe_usage_load(USAGE_PATH, 2, 4, r, 0) != MOE_OK) return 5;
  if (memcmp(c, r, sizeof c) != 0) return 6;
  if (moe_usage_load(USAGE_PATH, 4, 2, r, 0) != MOE_ERR_SHAPE) return 7;
  printf("ok\n");
  return 0;
}
""")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib._name)
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", f"-I{os.path.join(ROOT, 'include')}",
          f'-DUSAGE_PATH="{tmp_path / "u.bin"}"', str(src), f"-L{libdir}", "-lmoe",
          f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    subprocess.run(cc, check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
