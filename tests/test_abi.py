"""The C-ABI library builds, loads without a GPU and exports every entry point
declared in include/*.h (no compute calls: CPU only)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DECL = re.compile(r"^[A-Za-z_][\w \t\*]*?\b((?:nl|nls)_\w+)\s*\(", re.M)


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in DECL.finditer(text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def libpath():
    from neighbor_list_construction_b200 import build_lib
    return build_lib.build()


def test_headers_declare_the_path(libpath):
    names = declared_functions()
    for required in ("nl_sort_hilbert", "nl_build", "nl_skin_check", "nl_replay",
                     "nl_create", "nl_destroy", "nl_sync_status"):
        assert required in names


def test_every_declared_symbol_is_exported(libpath):
    lib = ctypes.CDLL(libpath)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_mirrors_the_header(libpath):
    from neighbor_list_construction_b200 import nl
    assert set(nl.EXPORTS) == set(declared_functions())
    for n in declared_functions():
        assert callable(getattr(nl, n))


def test_status_strings_without_gpu(libpath):
    from neighbor_list_construction_b200 import nl
    assert nl.nl_status_string(0) == "NL_OK"
    assert "capacity" in nl.nl_status_string(1)
    assert nl.nl_status_string(-2).startswith("NL_ERR_BOX")


def test_library_is_independent_of_the_oracle(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True,
                         text=True).stdout
    assert "oracle_" not in out


def test_sources_do_not_reference_the_oracle():
    for f in glob.glob(os.path.join(ROOT, "neighbor_list_construction_b200", "**", "*"),
                       recursive=True):
        if f.endswith((".cu", ".cuh", ".py", ".h")):
            text = open(f).read()
            assert "import oracle" not in text and "nl_oracle" not in text, f


def test_every_declaration_is_documented():
    """Each entry point in include/*.h has a comment block directly above it,
    or follows, with no blank line, a declaration of the same documented
    group: walking up over contiguous non-blank lines reaches a comment end."""
    undocumented = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        lines = text.split("\n")
        for m in DECL.finditer(text):
            j = text.count("\n", 0, m.start()) - 1
            ok = False
            while j >= 0 and lines[j].strip():
                if lines[j].rstrip().endswith("*/"):
                    ok = True
                    break
                j -= 1
            if not ok:
                undocumented.append(m.group(1))
    assert not undocumented, undocumented


NULL_CTX_PROBE = r'''
import ctypes, sys
sys.path.insert(0, sys.argv[1])
from neighbor_list_construction_b200 import nl
L = nl._lib
box = (ctypes.c_float * 3)(10, 10, 10)
dims = (ctypes.c_int32 * 3)(2, 2, 2)
calls = [
    L.nl_sort_hilbert(None, 10, None, box, None, None, None, None),
    L.nl_sort_morton(None, 10, None, box, None, None, None, None),
    L.nl_build(None, 10, None, box, 2.0, 0.5, 8, None, None, None),
    L.nl_build_rows(None, 10, 5, None, box, 2.0, 0.5, 8, None, None, None),
    L.nl_build_close(None, 10, None, box, 2.0, 0.5, 8, None, None, 1.0, None, None, None),
    L.nl_edge_features(None, 10, None, box, None, None, 8, None, None),
    L.nl_csr_offsets(None, 10, None, 8, None, None),
    L.nl_csr_fill(None, 10, None, None, 8, None, None, None, box, None, None),
    L.nl_skin_check(None, 10, None, box, 0.5, None, None, None),
    L.nl_replay(None, None, 4, 10, None, box, 2.0, 0.5, 8, None, None, None, None),
    L.nl_replay_resort(None, None, 4, 10, None, None, None, box, 2.0, 0.5, 8, None, None, None, None),
    L.nl_sync_status(None, None),
    L.nl_last_build_info(None, None),
    L.nl_profile_enable(None, 1),
    L.nl_profile_read(None, None, None, 4),
    L.nl_halo_mark(None, 10, None, box, dims, 0, None, None),
    L.nl_halo_needed(None, box, dims, None, None, None),
    L.nl_halo_count(None, 10, None, box, dims, None, 0, 2, None, None),
    L.nl_halo_fill(None, 10, None, box, dims, None, 0, 2, None, None, None, None, None),
    L.nl_map_ids(None, 10, 8, None, None, 10, None, None),
    L.nl_wait_selftest(None, 10, None),
]
h = ctypes.c_void_p()
bad_create = [L.nl_create(ctypes.byref(h), 10, 0), L.nl_create(ctypes.byref(h), -1, 8),
              L.nl_create(None, 10, 8)]
L.nl_destroy(None)
import json
print("NULLCTX" + json.dumps({"calls": calls, "bad_create": bad_create,
                              "counter": L.nl_step_counter(None)}))
'''


def test_null_context_and_bad_create_are_refused_without_a_gpu():
    """Every entry point refuses a NULL context with NL_ERR_ARG before any
    CUDA call (run in a child process, so a crash fails this test only);
    nl_create refuses bad sizes and a NULL handle; nl_destroy(NULL) is a
    no-op."""
    import sys
    out = subprocess.run([sys.executable, "-c", NULL_CTX_PROBE, ROOT], capture_output=True,
                         text=True, timeout=120)
    assert out.returncode == 0, out.stderr[-2000:]
    import json
    line = [ln for ln in out.stdout.splitlines() if ln.startswith("NULLCTX")][0]
    got = json.loads(line[len("NULLCTX"):])
    assert got["calls"] == [-1] * 21          # NL_ERR_ARG
    assert got["bad_create"] == [-1] * 3
    assert got["counter"] is None
