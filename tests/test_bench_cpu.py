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


def test_kernel_bytes_per_step(bench):
    n, B = 1 << 24, 16
    w = wl("sym", n, B)
    # the aggregate pass runs on x and on g: the method's bytes are the sorted
    # anchors, the permutation and the gathered rows; the design adds the sorted copy
    assert bench.kernel_bytes_per_step("sym_agg", w) == (2 * (8 + 64) * n, 2 * (8 + 128) * n)
    assert bench.kernel_bytes_per_step("sym_bwd", w) == ((8 + 64 + 4) * n, (8 + 64 * 3 + 4) * n)
    assert bench.kernel_bytes_per_step("radix_pass", w) == (8 * n, 60 * n)
    assert bench.kernel_bytes_per_step("no_such_kernel", w) is None
    # summed over the kernels, the method's bytes are the compulsory bytes less the
    # backward's second read of x (it reads the forward's saved sorted copy) plus
    # the second reads of the sorted anchors and permutation by the sweeps
    names = ("sym_agg", "sym_fwd", "sym_bwd", "radix_pass", "radix_hist")
    total = sum(bench.kernel_bytes_per_step(k, w)[0] for k in names)
    assert total == bench.compulsory_bytes(w) - 4 * B * n + 16 * n == 304 * n
    g = wl("gram", 3 << 20, 8, 65536)
    assert bench.kernel_bytes_per_step("large_accum", g) == ((8 + 64) * (3 << 20),) * 2  # paired v and g rows
    # both sorts of the Gram operator are radix sorts (k > 8192): the step's radix
    # bytes cover both
    assert bench.kernel_bytes_per_step("radix_pass", g) == (8 * ((3 << 20) + 65536), 60 * ((3 << 20) + 65536))
    h = wl("phased_transpose", 1 << 22, 128, 1024)
    assert bench.kernel_bytes_per_step("sort_small", h) == (12 * 1024, 12 * 1024)  # k <= 8192: counting sort
    one = wl("sym", 10 ** 9, 1)
    assert bench.kernel_bytes_per_step("unpermute_place", one) == (12 * 10 ** 9, 36 * 10 ** 9)


def test_roofline_of_the_dominant_kernel(bench):
    n, B = 1 << 24, 16
    w = wl("sym", n, B)
    steps = 10
    prof = {"sym_agg": (2 * steps, 2 * steps * 0.6), "sym_bwd": (steps, steps * 1.0), "radix_pass": (40, 5.0)}
    r = bench.roofline_of(prof, w, steps, "sym2p24", 6549.1, "measured")
    assert r["kernel"] == "sym_agg" and r["launches_per_step"] == 2
    assert r["algorithmic_bytes_per_launch"] == (8 + 64) * n
    assert r["design_bytes_per_launch"] == (8 + 128) * n
    assert abs(r["achieved"] - (8 + 64) * n / 0.6e-3 / 1e9) < 0.1
    assert abs(r["frac"] - r["achieved"] / 6549.1) < 1e-4 and r["design_frac"] > r["frac"]
    assert bench.roofline_of({}, w, steps, "sym2p24", 6549.1, "measured") is None


def test_reference_arm_config_matches(bench):
    w = wl("sym", 1 << 24, 16)
    c = bench.config_of(w, "sym2p24", 1)
    assert c == bench.config_of(w, "sym2p24", 1) and c["workload"] == "sym2p24" and c["B"] == 16
    assert "no flush" in c["l2"]


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
