"""The C ABI library loads, exports every function include/*.h declares, and rejects bad
arguments on the host before touching the GPU (these calls make no CUDA call)."""

import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from moe_expert_shuffling_b200 import build
    path = build.build()
    lib = ctypes.CDLL(path)
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_version.restype = ctypes.c_char_p
    return lib


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"^MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M))
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_plan", "moe_dispatch", "moe_combine", "moe_plan_create",
                     "moe_plan_query", "moe_plan_check", "moe_plan_destroy", "moe_last_error"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    from moe_expert_shuffling_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    declared = declared_functions()
    missing = declared - exported
    assert not missing, missing
    # nothing else of ours leaks out of the library
    ours = {s for s in exported if s.startswith("moe_")}
    assert ours == declared, ours ^ declared
    for name in declared:
        assert hasattr(lib, name)


def test_version(lib):
    assert b"sm_100a" in lib.moe_version()


def _plan(lib, N, k, E, R):
    h = ctypes.c_void_p(0)
    st = lib.moe_plan(ctypes.c_void_p(0), ctypes.c_void_p(0), N, k, E, R, ctypes.c_void_p(0),
                      ctypes.byref(h))
    return st, lib.moe_last_error().decode()


@pytest.mark.parametrize("N,k,E,R,msg", [
    (4, 2, 8, 3, "R must divide E"),
    (4, 33, 64, 4, "k must be in"),
    (4, 0, 8, 4, "k must be in"),
    (-1, 2, 8, 4, "N must be >= 0"),
    (4, 4, 2048, 4, "E must be in"),
    (4, 9, 8, 4, "E must be in"),
    (1 << 28, 8, 64, 4, "N*k must be < 2^31"),
    (4, 2, 8, 4, "must not be NULL"),       # valid shape, but no routing arrays
])
def test_plan_rejects_bad_arguments_on_host(lib, N, k, E, R, msg):
    st, err = _plan(lib, N, k, E, R)
    assert st == 1, err          # MOE_EINVAL
    assert msg in err


def test_null_plan_rejected(lib):
    assert lib.moe_dispatch(None, 0, None, 64, None, None, None, None) == 1
    assert b"plan" in lib.moe_last_error()
    assert lib.moe_combine(None, 64, None, None, None) == 1
    assert lib.moe_plan(None, None, 0, 1, 1, 1, None, None) == 1
    assert lib.moe_plan_query(None, None) == 1
    assert lib.moe_plan_check(None, None, None) == 1
    assert lib.moe_plan_create(4, 2, 8, 4, None) == 1


def test_destroy_null_is_noop(lib):
    assert lib.moe_plan_destroy(None) == 0


def test_tune_rejects_unknown_knob(lib):
    assert lib.moe_tune(99, 1) == 1
    assert lib.moe_tune(4, 1) == 1   # retired knobs
    assert lib.moe_tune(7, 1) == 1
    assert lib.moe_tune(0, -1) == 1
    assert lib.moe_tune(0, 0) == 0   # default restored


def test_python_binding_imports_and_knows_knobs():
    import moe_expert_shuffling_b200 as ms
    assert ms.version().startswith("moeshuffle")
    assert set(ms.KNOBS) >= {"dispatch_stages", "combine_stages"}
    with pytest.raises(TypeError):
        ms.moe_plan("not a tensor", None, 8, 4)


def test_product_has_no_oracle_dependency():
    """The CUDA library and its binding never import, link or call the oracle."""
    pkg = os.path.join(ROOT, "moe_expert_shuffling_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*"), recursive=True):
        if os.path.isfile(path) and path.endswith((".py", ".cu", ".cuh", ".h")):
            text = open(path).read()
            assert "oracle" not in text.lower(), path
    out = subprocess.run(["ldd", os.path.join(pkg, "libmoeshuffle.so")], capture_output=True,
                         text=True).stdout
    assert "oracle" not in out


def test_python_knobs_match_the_header(lib):
    """Every MOE_TUNE_* value in the header is a knob of the binding under the same name and
    number, and the library accepts each of them."""
    import moe_expert_shuffling_b200 as ms
    text = open(os.path.join(ROOT, "include", "moe_shuffle.h")).read()
    header = {m.group(1).lower(): int(m.group(2))
              for m in re.finditer(r"MOE_TUNE_([A-Z0-9_]+)\s*=\s*(\d+)", text)}
    assert header == ms.KNOBS
    for value in header.values():
        assert lib.moe_tune(value, 0) == 0


def test_wait_selftest_rejects_unknown_wait_on_host(lib):
    flags = ctypes.c_uint32(0)
    assert lib.moe_wait_selftest(7, None, ctypes.byref(flags)) == 1
    assert lib.moe_wait_selftest(0, None, None) == 1


def test_fused_call_rejects_null_plans_on_host(lib):
    args = [None, 0, None, 64, None, None, None, None, 64, None, None, 0, None]
    assert lib.moe_dispatch_combine(*args) == 1
    assert b"plan" in lib.moe_last_error()


@pytest.mark.parametrize("N,k,E,R", [
    (1 << 20, 8, 256, 32),          # far beyond the fixed scratch array
    (127 * 128 + 1, 8, 1024, 1024),  # one tile past the limit: (2049) * 128 > 262144 words
    (907 * 128 + 1, 8, 256, 32),     # one tile past the limit: 289 * 908 > 262144 words
])
def test_noalloc_rejects_more_tokens_than_its_scratch_holds(lib, N, k, E, R):
    """The size limit of moe_plan_noalloc is checked on the host before anything else; no
    array is passed, so even a broken check could not launch a kernel."""
    lib.moe_plan_noalloc.restype = ctypes.c_int
    st = lib.moe_plan_noalloc(None, N, k, E, R, *([None] * 11), None)
    assert st == 1
    assert b"scratch" in lib.moe_last_error()


def test_plan_create_ex_rejects_unknown_flags(lib):
    h = ctypes.c_void_p(0)
    assert lib.moe_plan_create_ex(4, 2, 8, 4, 1, ctypes.c_uint32(2), ctypes.byref(h)) == 1
    assert b"flags" in lib.moe_last_error()
    assert not h.value


def test_ranks_started_together_build_the_library_once(tmp_path):
    """Two processes that need the library at once (two ranks of one node) compile it once:
    the second waits on the build lock and then finds the first one's library fresh.  The
    compiler is a stand-in script, so this runs without nvcc or a GPU."""
    count = tmp_path / "compiles"
    fake = tmp_path / "fake_nvcc"
    fake.write_text(
        "#!/bin/bash\n"
        f"echo run >> {count}\n"
        "sleep 1\n"
        "out=''\n"
        "while [ $# -gt 0 ]; do if [ \"$1\" = -o ]; then out=$2; fi; shift; done\n"
        "echo library > \"$out\"\n")
    fake.chmod(0o755)
    out = tmp_path / "libtest.so"
    code = ("import sys; sys.path.insert(0, %r); from moe_expert_shuffling_b200 import build; "
            "build.build(out=%r)" % (ROOT, str(out)))
    env = dict(os.environ, NVCC=str(fake))
    procs = [subprocess.Popen(["python", "-c", code], env=env) for _ in range(2)]
    assert all(p.wait(timeout=120) == 0 for p in procs)
    assert count.read_text().splitlines() == ["run"]
    assert out.read_text() == "library\n"
    assert not list(tmp_path.glob("libtest.so.tmp*"))
