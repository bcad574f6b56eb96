"""Host-side helpers of bench.py: the roofline's algorithmic bytes, the peak
it divides by, and when an ncu traffic record is trusted. No GPU needed."""
import json
import os

import pytest

import bench
import workloads as wl


def test_algorithmic_bytes_by_hand():
    """Tiny workload (4 sequences, 4 heads, head_dim 64, bs 16): every context
    token's K and V rows, the query and output rows, and 4 bytes per
    block-table entry read; the partly filled last block is not rounded up."""
    st = wl.tiny()
    H, D, bs = st.num_heads, st.head_dim, st.block_size
    ctx = [int(c) for c in st.context_lens]
    kv = sum(c * H * D * 2 * 2 for c in ctx)                 # K + V, f16
    qo = st.num_seqs * H * D * 2 * 2                         # query + output, f16
    table = sum((c + bs - 1) // bs for c in ctx) * 4
    ab = bench.algorithmic_bytes(st)
    assert ab["kv"] == kv
    assert ab["total"] == kv + qo + table


def test_algorithmic_bytes_fp8_counts_row_scales():
    """fp8 rows: head_dim code bytes plus a 4-byte scale per row."""
    st = wl.tiny(dtype="fp8")
    H, D = st.num_kv_heads, st.head_dim
    kv = sum(int(c) * H * (D + 4) * 2 for c in st.context_lens)
    assert bench.algorithmic_bytes(st)["kv"] == kv


def test_measured_peak_falls_back_without_the_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak() == (bench.FALLBACK_PEAK_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6425.6}))
    assert bench.measured_peak() == (6425.6, "measured")


def _fake_root(tmp_path, kernel_text):
    csrc = tmp_path / "paged_kv_cache_417_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "decode.cuh").write_text(kernel_text)
    (csrc / "ptx.cuh").write_text("// ptx helpers\n")
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_record_is_used_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    """A record carries a hash of the kernel's sources; once a source changes
    the record is void (the bench then reports traffic null)."""
    csrc = _fake_root(tmp_path, "// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash(("decode.cuh", "ptx.cuh"))
    rec = {"llama7b_layer": {"sources": ["decode.cuh", "ptx.cuh"],
                             "kernel_source_hash": h, "dram_bytes_per_launch": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("llama7b_layer") == 123
    assert bench.recorded_traffic("long_context") is None          # no record
    (csrc / "decode.cuh").write_text("// kernel v2\n")
    assert bench.recorded_traffic("llama7b_layer") is None         # stale


def test_traffic_keys_name_the_variant():
    class A:
        config, kv_dtype, kv_heads, seqs = "llama7b_layer", "f16", 0, 0
    a = A()
    assert bench.traffic_key(a) == "llama7b_layer"
    a.kv_dtype, a.kv_heads = "fp8", 8
    assert bench.traffic_key(a) == "llama7b_layer_fp8_kvh8"


def test_committed_traffic_records_are_well_formed():
    """Every committed record names existing sources, a 16-hex-digit hash and a
    positive byte count within a few per cent of the config's algorithmic
    bytes (DRAM traffic far above them would mean re-reads)."""
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as f:
        recs = json.load(f)
    csrc = os.path.join(bench.ROOT, "paged_kv_cache_417_b200", "csrc")
    for key, rec in recs.items():
        for src in rec["sources"]:
            assert os.path.exists(os.path.join(csrc, src)), (key, src)
        assert len(rec["kernel_source_hash"]) == 16
        int(rec["kernel_source_hash"], 16)
        assert rec["dram_bytes_per_launch"] > 0
    st = wl.llama_layer(seed=bench.SEEDS["llama7b_layer"])
    ratio = recs["llama7b_layer"]["dram_bytes_per_launch"] / bench.algorithmic_bytes(st)["total"]
    assert 0.99 < ratio < 1.05


def test_job_throughput_counts_every_rank():
    # 2 ranks x 96 sequences x 10 steps in 5 ms of the slowest rank
    assert bench.job_throughput(2, 96, 10, 5.0) == pytest.approx(2 * 96 * 10 / 5e-3)


def test_other_configs_name_real_workloads():
    """The short extra runs of a default bench line use workloads and flags
    the script accepts."""
    for name, extra, steps in bench.OTHER_CONFIGS:
        assert steps > 0
        if "--config" in extra:
            assert extra[extra.index("--config") + 1] in bench.WORKLOADS, name
        if "--kv-dtype" in extra:
            assert extra[extra.index("--kv-dtype") + 1] in ("f16", "bf16", "fp8"), name
