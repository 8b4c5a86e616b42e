"""Host-side checks of bench.py's bookkeeping (no GPU): the kernel-source hash that keys the
recorded DRAM counters ignores comments and blank lines but sees every code change."""
import importlib.util
import os

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


SRC = '''// header comment
#include "x.cuh"
/* block
   comment */
__global__ void k(int* p) {   // trailing comment
    const char* s = "not // a comment";

    p[0] = '/';  /* inline */ p[1] = 2;
}
'''


def test_comments_and_blank_lines_do_not_count(bench):
    a = bench._code_only(SRC)
    b = bench._code_only(SRC.replace("// header comment", "// another header").replace("inline", "other")
                         .replace("\n\n", "\n\n\n"))
    assert a == b
    assert "not // a comment" in a and "'/'" in a and "header" not in a and "block" not in a


def test_code_changes_count(bench):
    a = bench._code_only(SRC)
    assert bench._code_only(SRC.replace("p[1] = 2", "p[1] = 3")) != a
    assert bench._code_only(SRC.replace('"not // a comment"', '"not // a remark"')) != a


def test_recorded_traffic_is_keyed_on_the_current_sources(bench):
    # every record in profiles/traffic.txt is either current (a float) or reported as null
    for kind in ("fwd_main", "dx_main"):
        v = bench.recorded_traffic(kind)
        assert v is None or v > 0
