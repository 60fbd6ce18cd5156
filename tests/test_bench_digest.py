"""The kernel-source digest that ties recorded ncu counters (profiles/traffic.json)
to the sources: blind to comments, sensitive to code."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_strip_keeps_code_and_literals():
    src = ('int a = 1;  // one\n/* block\n comment */ int b = 2;\n\n'
           'const char* s = "x // y /* z */";\nchar q = \'"\'; char e = \'\\\'\'; // end\n')
    out = bench.strip_c_comments(src)
    assert "one" not in out and "block" not in out and "end" not in out
    assert '"x // y /* z */"' in out
    assert "char q = '\"'; char e = '\\'';" in out
    assert "int a = 1;" in out and "int b = 2;" in out
    assert "\n\n" not in out


def _tree(tmp_path, kernel_src):
    csrc = tmp_path / "mixture_experts_projections_b200" / "csrc"
    csrc.mkdir(parents=True, exist_ok=True)
    (tmp_path / "include").mkdir(exist_ok=True)
    (csrc / "k.cu").write_text(kernel_src)
    shutil.copy(os.path.join(ROOT, "include", "rom.h"), tmp_path / "include" / "rom.h")
    return str(tmp_path)


def test_digest_ignores_comments_not_code(tmp_path):
    base = "// kernel\n__global__ void k(float* x) { x[0] = 1.0f; }\n"
    d0 = bench.csrc_digest(_tree(tmp_path, base))
    d1 = bench.csrc_digest(_tree(tmp_path, "// a reworded comment\n/* more */\n" + base))
    d2 = bench.csrc_digest(_tree(tmp_path, base.replace("1.0f", "2.0f")))
    assert d0 == d1
    assert d0 != d2


def test_recorded_traffic_only_for_matching_sources():
    """bench.py reports a recorded DRAM traffic figure only while the digest
    recorded with it matches the sources it runs."""
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    cur = bench.csrc_digest()
    for w, ent in t.items():
        want = ent["dram_bytes_per_launch"] if ent["csrc_sha256"] == cur else None
        assert bench.profiled_traffic(w) == want, w
    assert bench.profiled_traffic("no_such_workload") is None
