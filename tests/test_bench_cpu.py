"""Host logic of bench.py that the reported numbers depend on (no GPU): the
compulsory and per-kernel algorithmic byte counts, the DRAM-traffic records keyed
by the kernel's sources, and the summary of the clock samples taken during the
timed region."""
import importlib.util
import os
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def wl(op, n, B, k=0):
    return SimpleNamespace(op=op, n=n, B=B, k=k)


def test_compulsory_bytes_of_the_symmetric_step(bench):
    n, B = 1 << 24, 16
    # sort: a in, a_sorted + perm out; forward: a_sorted, perm, x in, y out;
    # backward: a_sorted, perm, x, g in, gx, ga out
    expect = (4 + 8) * n + (8 * n + 4 * n * B * 2) + (8 * n + 4 * n * B * 3 + 4 * n)
    assert bench.compulsory_bytes(wl("sym", n, B)) == expect == 5905580032


def test_kernel_bytes_per_launch(bench):
    w = wl("sym", 1 << 24, 16)
    assert bench.kernel_bytes_per_launch("sym_agg", w) == (8 + 64 + 64) * (1 << 24)
    assert bench.kernel_bytes_per_launch("sym_bwd", w) == (8 + 64 * 3 + 4) * (1 << 24)
    assert bench.kernel_bytes_per_launch("no_such_kernel", w) is None
    g = wl("gram", 3 << 20, 8, 65536)
    assert bench.kernel_bytes_per_launch("large_accum", g) == (8 + 64) * (3 << 20)  # paired v and g rows


def test_traffic_records_follow_the_kernel_sources(bench, tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    h = bench.source_hash("sym_agg")
    (prof / "dram_traffic.txt").write_text(
        "# comment\n"
        f"traffic sym_agg sym2p24 123 {h}\n"
        "traffic sym_fwd sym2p24 456 0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the hash is of the sources under ROOT: point it back at the repository's
    monkeypatch.setattr(bench, "source_hash", lambda k, _h=h: _h if k.startswith("sym_") else "x")
    assert bench.recorded_traffic("sym_agg", "sym2p24") == 123.0
    assert bench.recorded_traffic("sym_fwd", "sym2p24") is None   # taken on other sources
    assert bench.recorded_traffic("sym_agg", "sym1e9") is None    # other workload


def test_source_hash_depends_on_the_kernel_file(bench):
    assert bench.source_hash("sym_agg") == bench.source_hash("sym_bwd")      # both in sym.cu
    assert bench.source_hash("sym_agg") != bench.source_hash("radix_pass")   # sym.cu vs sort.cu
    assert len(bench.source_hash("large_accum")) == 16


def test_clock_summary(bench, tmp_path):
    csv = tmp_path / "clocks.csv"
    csv.write_text(
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
        "1, 1200, 1965, 300.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
        "0, 1950, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
        "0, 1965, 1965, 995.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
        "garbage line\n")
    s = bench.summarize_clocks(str(csv), 0)
    assert s["samples"] == 3 and s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clocks(str(tmp_path / "missing.csv"), 0)["samples"] == 0


def test_comment_edits_leave_the_source_hash_alone(bench):
    a = 'int a; // one\n/* two\n lines */ const char* s = "x // kept"; float f;'
    b = 'int a;   // changed\n/* other */ const char* s = "x // kept";\nfloat f;'
    assert bench._code_only(a) == bench._code_only(b) == 'int a; const char* s = "x // kept"; float f;'
    assert bench._code_only('x = "a\\"b // in string"; y; // gone') == 'x = "a\\"b // in string"; y;'
