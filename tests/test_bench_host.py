"""Host-side logic of bench.py on CPU: the algorithmic byte counts, the
measured-traffic file and its source digests, the whole-job value and the
reference arm's output line."""
import json
import os
import subprocess
import sys

import pytest

import bench


def test_algorithmic_bytes_per_element():
    # in + out bytes per element: bf16 in, half a byte of codes and a
    # scale byte per 32 out (the double quantizer writes both layouts)
    assert bench.BYTES_PER_ELEM["quant_rows_rne"] == 2 + 0.5 + 1 / 32
    assert bench.BYTES_PER_ELEM["double_quant"] == 2 + 2 * (0.5 + 1 / 32)
    assert bench.BYTES_PER_ELEM["dequant_rows"] == 0.5 + 1 / 32 + 2
    assert bench.BYTES_PER_ELEM["osc_step"] == 28   # 4 arrays read, 3 written
    for op, per in bench.READ_BYTES_PER_ELEM.items():
        assert per <= bench.BYTES_PER_ELEM[op]
    assert bench.alg_bytes("double_quant") == 3.0625 * 8192 * 28672
    assert bench.STEP_BYTES == sum(bench.alg_bytes(op) for op in bench.BYTES_PER_ELEM)


def test_job_value_counts_every_rank_over_the_slowest():
    # 2 ranks, 1 GB a step each, 10 steps in 5 ms (the slower rank): 4000 GB/s
    assert abs(bench.job_gbs(2, 1e9, 10, 5.0) - 4000.0) < 1e-9


def test_measured_traffic_follows_the_source_digest(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    digest = bench.kernel_source_digest("double_quant")
    (prof / "dram_traffic.txt").write_text(
        "# comment\n"
        "double_quant 470000000 220000000 src=%s\n"
        "quant_cols_sr 1 2 src=000000000000\n" % digest)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the source files are looked up under ROOT: point the digest at the
    # real tree while the profile file comes from tmp
    real = os.path.dirname(os.path.abspath(bench.__file__))
    monkeypatch.setattr(bench, "kernel_source_digest", lambda op: _digest_in(real, op))
    assert bench.measured_traffic("double_quant") == (470000000.0, 220000000.0)
    assert bench.measured_traffic("quant_cols_sr") is None     # stale digest
    assert bench.measured_traffic("osc_step") is None          # no line


def _digest_in(root, op):
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(root, "mxfp4_block_quantization_quantizer_b200", "csrc")
    for name in bench.OP_SOURCES[op]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:12]


def test_committed_traffic_reads_no_more_than_it_must():
    """Each current line of profiles/dram_traffic.txt (captured from the
    kernel sources as they are now; a stale one reads null in the bench and
    is skipped here) reads within 10% of the algorithmic read bytes."""
    current = 0
    for op in ("quant_rows_rne", "quant_cols_sr", "double_quant", "dequant_rows",
               "rht_quant_sr", "osc_step"):
        got = bench.measured_traffic(op)
        if got is None:
            continue
        current += 1
        read, write = got
        ratio = read / (bench.READ_BYTES_PER_ELEM[op] * bench.OP_ELEMS[op])
        assert 0.99 < ratio < 1.1, (op, ratio)
    if current == 0:
        pytest.skip("no traffic line matches the current kernel sources")


def test_reference_arm_prints_one_json_line():
    root = os.path.dirname(os.path.abspath(bench.__file__))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
