"""The ncu summaries under profiles/ that bench.py reads: every recorded per-call DRAM
traffic line parses and names kernel sources that exist."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PAT = re.compile(r"<!-- traffic (\w+) bytes_per_call=(\d+) sources=([\w./,]+) sha256=([0-9a-f]{64}) -->")


def test_traffic_lines_parse_and_name_existing_sources():
    found = 0
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for m in PAT.finditer(open(path).read()):
            found += 1
            assert int(m.group(2)) > 0
            for f in m.group(3).split(","):
                assert os.path.exists(os.path.join(ROOT, "decoder_only_transformer_train_b200", f)), f
    assert found > 0


def test_bench_reports_null_traffic_for_unknown_class():
    import bench
    value, note = bench.recorded_traffic("no_such_class")
    assert value is None and note
