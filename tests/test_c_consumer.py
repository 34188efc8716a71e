"""The C ABI from C: tests/c_consumer.c includes include/moe_b200.h as C99
(-Wall -Wextra -pedantic -Werror), links libmoe_b200.so and calls the entry
points that need no GPU.  Its size queries must equal the Python binding's,
and the argument structs' sizes and field offsets must equal the binding's
ctypes mirrors (a field added on one side only would shift every later one)."""
import ctypes
import os
import shutil
import subprocess

import pytest

import mixture_experts_expert_moe_b200 as m

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GCC = shutil.which("gcc")


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    if GCC is None:
        pytest.fail("gcc is required to build the C consumer")
    lib_dir = os.path.dirname(m.LIB_PATH)
    if not os.path.exists(m.LIB_PATH):
        pytest.fail(f"{m.LIB_PATH} is missing: build it first")
    exe = str(tmp_path_factory.mktemp("c_consumer") / "c_consumer")
    cmd = [GCC, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_consumer.c"), "-o", exe, f"-L{lib_dir}", "-l:" + os.path.basename(m.LIB_PATH),
           f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, f"exit {r.returncode}: {r.stdout}{r.stderr}"
    out = {}
    for line in r.stdout.splitlines():
        parts = line.split()
        if parts[0] in ("sizeof", "offset"):     # "sizeof <struct> N", "offset <struct> <field> N"
            out[" ".join(parts[:-1])] = parts[-1:]
        else:                                    # "<name> v1 [v2 ...]"
            out[parts[0]] = parts[1:]
    return out


def test_c_size_queries_match_the_binding(c_output):
    P, NB, ws = (int(v) for v in c_output["align"])
    assert (P, NB, ws) == m.align_sort_sizes(16384, 8, 256, 64)
    lib = m.load_library()
    a = m.FfnArgs(T=2048, H=7168, I=2048, E=256, k=8, block_size=64, wdtype=m.MOE_BF16)
    n = ctypes.c_size_t()
    assert lib.moe_ffn_workspace(ctypes.byref(a), ctypes.byref(n)) == 0
    assert int(c_output["ffn_ws"][0]) == n.value
    f = m.ForwardArgs(T=2048, H=7168, I=2048, E=256, k=8, block_size=64, wdtype=m.MOE_BF16, out_dtype=m.MOE_BF16)
    assert lib.moe_forward_workspace(ctypes.byref(f), ctypes.byref(n)) == 0
    assert int(c_output["forward_ws"][0]) == n.value


@pytest.mark.parametrize("struct,mirror", [("moe_ffn_args", m.FfnArgs), ("moe_forward_args", m.ForwardArgs),
                                           ("moe_backward_args", m.BackwardArgs)])
def test_struct_layouts_match_the_ctypes_mirrors(c_output, struct, mirror):
    assert int(c_output[f"sizeof {struct}"][0]) == ctypes.sizeof(mirror)
    for key, val in c_output.items():
        parts = key.split()
        if parts[0] == "offset" and parts[1] == struct:
            assert int(val[0]) == getattr(mirror, parts[2]).offset, key
