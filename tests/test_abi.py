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
