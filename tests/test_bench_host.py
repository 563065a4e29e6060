"""Host-side logic of bench.py that needs no GPU: the DRAM-traffic records of the committed ncu
summary are tied to each kernel's own source files, and go stale (null) exactly when those
files change."""
import json
import os
import shutil

import bench


def _tree(tmp_path):
    csrc = tmp_path / "gated_deltanet_token_b200" / "csrc"
    shutil.copytree(os.path.join(bench.ROOT, "gated_deltanet_token_b200", "csrc"), csrc)
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_record_follows_its_kernel_sources(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {k: {"dram_bytes_per_launch": 1000 + i, "src_sha": bench.source_sha(files)}
           for i, (k, files) in enumerate(sorted(bench.KERNEL_SOURCES.items()))}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    for k in bench.KERNEL_SOURCES:
        assert bench.ncu_traffic(k) == rec[k]["dram_bytes_per_launch"]
    # a change to the decode kernel's header stales the decode record only
    with open(csrc / "k_decode.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.ncu_traffic("decode") is None
    for k in ("chunk_prep_tc", "chunk_scan_tc_norm", "chunk_phaseB_simt", "decode_multi"):
        assert bench.ncu_traffic(k) == rec[k]["dram_bytes_per_launch"]
    # a change to a header every kernel includes stales them all
    with open(csrc / "gdn_common.cuh", "a") as f:
        f.write("\n// edited\n")
    assert all(bench.ncu_traffic(k) is None for k in bench.KERNEL_SOURCES)


def test_unknown_kernel_or_missing_summary_reads_null(tmp_path, monkeypatch):
    _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("chunk_scan_tc_norm") is None  # no summary file
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps({"k_other": {"src_sha": "x"}}))
    assert bench.ncu_traffic("k_other") is None

