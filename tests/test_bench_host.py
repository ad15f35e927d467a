"""Host-side logic of bench.py that needs no GPU: the source-hash gate on the
roofline traffic figure, and the per-step inputs of the MTP-verify workload."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _table(tmp_path, kernel, files, sha, nbytes):
    p = tmp_path / "traffic.txt"
    p.write_text(f"# kernel sources sha256 bytes\n{kernel} {','.join(files)} {sha} {nbytes} some workload\n")
    return str(p)


def test_traffic_used_only_while_sources_match(tmp_path):
    files = ["ffn_decode.cu", "dequant.cuh"]
    sha = bench.source_sha256(files)
    assert bench.measured_traffic("k", _table(tmp_path, "k", files, sha, 123456)) == 123456.0
    stale = ("0" if sha[0] != "0" else "1") + sha[1:]
    assert bench.measured_traffic("k", _table(tmp_path, "k", files, stale, 123456)) is None
    assert bench.measured_traffic("other", _table(tmp_path, "k", files, sha, 1)) is None
    assert bench.measured_traffic("k", str(tmp_path / "missing.txt")) is None


def test_source_hash_sees_code_not_comments():
    # comment and layout edits keep a captured traffic figure; a code edit drops it
    base = "int f(int a) {  // add one\n  return a + 1; /* done */\n}\n"
    reworded = "/* header */\nint f(int a) { // increment\n\n    return a + 1;\n}"
    changed = "int f(int a) {  // add one\n  return a + 2; /* done */\n}\n"
    assert bench._code_only(base) == bench._code_only(reworded)
    assert bench._code_only(base) != bench._code_only(changed)
    assert "add one" not in bench._code_only(base)


def test_committed_traffic_table_parses():
    # every row names existing sources and a positive byte count
    with open(os.path.join(ROOT, "profiles", "roofline_traffic.txt")) as fh:
        rows = [l.split() for l in fh if l.strip() and not l.startswith("#")]
    assert rows
    for f in rows:
        assert len(f[2]) == 64 and float(f[3]) > 0
        bench.source_sha256(f[1].split(","))  # the files exist


def test_mtp_verify_inputs_are_correlated_drafts():
    cfg = bench.WORKLOADS["mtp_verify"]
    x = bench.step_inputs(cfg, "mtp_verify", 3, 0, "cpu")
    assert x.shape == (3, cfg.T, cfg.H) and x.dtype == torch.bfloat16
    xf = x.float()
    d = (xf[:, 1:] - xf[:, :1]).std().item()
    assert 0.03 < d < 0.12            # drafts differ from each other by ~0.05 * sqrt(2)
    assert xf.std().item() > 0.8      # around a common N(0, 1) draft


def test_decode_inputs_are_independent_tokens():
    cfg = bench.WORKLOADS["small_batch"]
    x = bench.step_inputs(cfg, "small_batch", 2, 0, "cpu").float()
    assert x.shape == (2, cfg.T, cfg.H)
    assert (x[:, 1:] - x[:, :1]).std().item() > 1.0
