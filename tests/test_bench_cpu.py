"""bench.py's accounting on CPU: the algorithmic bytes behind the roofline figures."""
import bench
import synth


def test_stage_bytes_at_256k():
    wl = synth.workload("ctx256k_12l")
    n = 255_182                                   # one decode step after the 255,181-token prefill
    b = bench.stage_bytes(wl, n)
    B = n // 4                                    # 63,795 completed blocks
    assert B == 63_795
    # scan: every pooled row once (B x d x f16), the scores out, the query and weights in
    assert b["index_scan"] == B * 128 * 2 + B * 4 + 16 * (128 * 2 + 4)
    assert B * 128 * 2 == 16_331_520
    # attention: 4*512 + (n mod 4) = 2,050 cells x 4 KV heads x (K + V) x 128 f16, plus ids, q, out
    cells = 4 * 512 + n % 4
    assert cells == 2_050
    assert b["sparse_attend"] == 512 * 4 + cells * 2 * 128 * 2 * 4 + 32 * 128 * (2 + 4)
    assert cells * 2 * 128 * 2 * 4 == 4_198_400
    # selection: the score table and the selected ids
    assert b["block_topk"] == B * 4 + 512 * 4


def test_stage_bytes_fp8_rows_carry_their_scale():
    wl = synth.workload("ctx256k_12l")
    n = 255_182
    cells = 4 * 512 + n % 4
    b8 = bench.stage_bytes(wl, n, kv_fp8=True)
    assert b8["sparse_attend"] == 512 * 4 + cells * 2 * (128 + 4) * 4 + 32 * 128 * (2 + 4)
    assert b8["index_scan"] == bench.stage_bytes(wl, n)["index_scan"]   # the indexer stays f16


def test_measured_peaks_have_a_source():
    peak, src = bench.measured_peaks()
    assert peak > 1000 and isinstance(src, str) and src


def test_stage_bytes_8bit_pooled_keys_carry_their_scale():
    wl = synth.workload("ctx256k_12l")
    n = 255_182
    B = n // 4
    b8 = bench.stage_bytes(wl, n, pooled_fp8=True)
    # every pooled row once as d code bytes plus its f32 scale, the scores out, the query in
    assert b8["index_scan"] == B * (128 + 4) + B * 4 + 16 * (128 * 2 + 4)
    assert b8["sparse_attend"] == bench.stage_bytes(wl, n)["sparse_attend"]   # attention unchanged


def test_ncu_traffic_is_tied_to_the_sources(tmp_path, monkeypatch):
    """The counters file's traffic is reported only while the hash of the kernel's sources
    matches; an edited source makes it null."""
    import json
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    h = hashlib.sha256(b"kernel v1").hexdigest()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_counters.json").write_text(json.dumps(
        {"kernels": {"index_scan": {"sources": ["k.cu"], "dram_bytes": 123, "sources_sha256": h}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("index_scan") == 123
    src.write_text("kernel v2")
    assert bench.ncu_traffic("index_scan") is None
    assert bench.ncu_traffic("block_topk") is None
