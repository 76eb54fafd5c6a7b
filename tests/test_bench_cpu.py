"""Host logic of bench.py that needs no GPU: the DRAM traffic a bench line reports comes
from a committed ncu summary only while the decode kernels' sources are the ones that
summary was taken on."""
import os
import shutil

import bench

SOURCES = ("decode_attention.cuh", "decode_attention_mma.cuh", "decode_attention_i8.cuh", "pkv_device.cuh")


def _fake_root(tmp_path):
    csrc = tmp_path / "paged_kv_cache_460_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in SOURCES:
        shutil.copy(os.path.join(bench.ROOT, "paged_kv_cache_460_b200", "csrc", name), csrc / name)
    (tmp_path / "profiles").mkdir()
    return tmp_path


def _write_profile(root, name, digest, dram_bytes):
    (root / "profiles" / ("decode_attention_%s.md" % name)).write_text(
        "# a summary\n\n- kernel_source_digest: `%s`\n- dram_bytes_per_attention_call: %d\n- other: 1\n"
        % (digest, dram_bytes))


def test_traffic_is_read_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    root = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    digest = bench.kernel_source_digest()
    _write_profile(root, "w", digest, 123456789)
    _write_profile(root, "int8_w", digest, 98765)
    assert bench.profiled_traffic("w") == 123456789
    assert bench.profiled_traffic("w", "int8") == 98765
    assert bench.profiled_traffic("other") is None               # no summary for this workload
    with open(root / "paged_kv_cache_460_b200" / "csrc" / "decode_attention_i8.cuh", "ab") as f:
        f.write(b"\n")                                            # any change to a kernel source ...
    assert bench.kernel_source_digest() != digest
    assert bench.profiled_traffic("w") is None                    # ... retires the old counters
    assert bench.profiled_traffic("w", "int8") is None


def test_committed_decode_summaries_carry_digest_and_traffic():
    names = [n for n in os.listdir(os.path.join(bench.ROOT, "profiles")) if n.startswith("decode_attention_")]
    assert names
    for n in names:
        with open(os.path.join(bench.ROOT, "profiles", n)) as f:
            text = f.read()
        assert "- kernel_source_digest: `" in text, n
        assert "- dram_bytes_per_attention_call: " in text, n


def test_cpu_baseline_times_both_legs_on_the_same_pairs():
    import synth
    s = synth.spec("tiny")
    res = bench.time_oracle_sample(s, 0.05, seed=3)
    assert res["single"] > 0 and res["all"] > 0
    assert res["threads"] >= 1 and res["cores_available"] >= 1 and res["cpu_model"]
    entry = bench.cpu_baseline_entry(res, "GB/s")
    assert entry["kind"] == "oracle" and entry["cores"] == res["threads"]
    assert entry["value"] == res["all"] and entry["single_thread"]["cores"] == 1


def test_reference_arm_prints_one_line(capsys):
    import json
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"]) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
