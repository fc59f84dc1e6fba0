"""Host-side pieces of bench.py that decide what the JSON line reports: the
code fingerprint that keys the committed DRAM-traffic records (it must follow
the code and ignore comments and layout), the traffic lookup itself, and the
packing of the end-to-end step's inputs into one buffer."""
import json
import os

import numpy as np
import pytest

import bench


def _write(tmp_path, name, text):
    p = tmp_path / name
    p.write_text(text)
    return str(p)


def test_fingerprint_ignores_comments_and_whitespace(tmp_path):
    a = _write(tmp_path, "a.cu", "int f(int x) {\n  return x + 1; // add one\n}\n/* block\n comment */\n")
    b = _write(tmp_path, "b.cu", "// header\nint f(int x)\n{\n\treturn x + 1;\n}\n")
    assert bench.code_fingerprint(a) == bench.code_fingerprint(b)


def test_fingerprint_follows_the_code(tmp_path):
    a = _write(tmp_path, "a.cu", "int f(int x) { return x + 1; }\n")
    b = _write(tmp_path, "b.cu", "int f(int x) { return x + 2; }\n")
    assert bench.code_fingerprint(a) != bench.code_fingerprint(b)


def test_fingerprint_keeps_comment_markers_inside_strings(tmp_path):
    a = _write(tmp_path, "a.cu", 'const char *s = "a // b";\n')
    b = _write(tmp_path, "b.cu", 'const char *s = "a ";\n')
    assert bench.code_fingerprint(a) != bench.code_fingerprint(b)


def test_traffic_lookup_follows_the_fingerprint():
    """A committed record is reported while its source's code is the one the
    capture was taken on, and null once the code has changed."""
    recs = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    assert recs
    for key, rec in recs.items():
        kernel, rest = key.split("@")
        workload, layout = rest.split(":")
        src = os.path.join(bench.ROOT, rec["source"])
        fresh = bench.code_fingerprint(src) == rec["code_sha256"]
        assert bench.traffic_record(kernel, workload, layout) == (rec["bytes_per_launch"] if fresh else None), key
    assert bench.traffic_record("hash_keys", "no_such_workload", "bytes") is None


def test_packed_inputs_round_trip():
    arrays = [np.arange(5, dtype=np.int16), np.arange(7, dtype=np.int32) - 3, np.linspace(0, 1, 3, dtype=np.float32)]
    buf = bench._pack_host(arrays)
    off = 0
    for a in arrays:
        assert off % 256 == 0
        np.testing.assert_array_equal(buf[off:off + a.nbytes].view(a.dtype), a)
        off += (a.nbytes + 255) // 256 * 256
    assert buf.nbytes == off


def test_both_arms_report_the_same_config():
    """The GPU arm and the reference arm print config_of(workload) unchanged:
    it names the workload only (no launch mode or kernel path)."""
    import workloads
    w = workloads.get(bench.DEFAULT_WORKLOAD)
    cfg = bench.config_of(w)
    assert cfg["workload"] == "ragged16" and cfg["code_layout"] == "planes"
    assert not {"launch", "decode_path", "mode"} & set(cfg)
    assert cfg == bench.config_of(workloads.get("ragged16"))


def test_step_contents_per_workload():
    """Only the 16k Llama-shaped layer hashes every cached key inside the
    step; elsewhere the key-hash build is timed apart."""
    import workloads
    assert bench.hash_in_step(workloads.get("llama8b_16k"))
    for name in ("ragged16", "batch8_64k", "batch4_128k", "ragged4", "tiny"):
        assert not bench.hash_in_step(workloads.get(name))


def test_decode_bytes_hand_count():
    """Two sequences of 100 and 3 tokens, K=8, L=75, sink 4 + window 64,
    2 kv heads, 10 union rows: codes 103 x 2 x 75 B; exact rows: 68 for the
    long sequence (4 + 64) and all 3 of the short one, per kv head."""
    import workloads
    w = workloads.get("tiny").with_(n_kv_heads=2, n_q_heads=2)
    total, codes, d_rows = bench.decode_bytes(w, np.array([100, 3]), 10)
    assert codes == 103 * 2 * 75
    assert d_rows == (68 + 3) * 2
    assert total == codes + (10 + d_rows) * 512
    # int8 keys: 128 B of K, its 16-byte record and 256 B of V per row
    total8, codes8, d_rows8 = bench.decode_bytes(w, np.array([100, 3]), 10, "int8")
    assert (codes8, d_rows8) == (codes, d_rows)
    assert total8 == codes + (10 + d_rows) * (128 + 16 + 256)


def test_code_layout_of_follows_the_library_rule():
    """The bench reports the layout the library picks for MP_CODES_AUTO:
    bit planes for the large K = 8 workloads and K = 10, byte codes for the
    16k-token layer."""
    import workloads
    assert bench.code_layout_of(workloads.get("ragged16")) == "planes"
    assert bench.code_layout_of(workloads.get("ragged4")) == "planes"
    assert bench.code_layout_of(workloads.get("batch8_64k")) == "planes"
    assert bench.code_layout_of(workloads.get("llama8b_16k")) == "bytes"
    assert bench.code_layout_of(workloads.get("ragged16").with_(code_layout="bytes")) == "bytes"


def test_oracle_sample_units_spread_over_the_batch():
    import workloads
    w = workloads.get("ragged16")
    smp = bench.OracleSample(w)
    assert smp.units == [(0, 0), (4, 1), (8, 2), (12, 3)]
    assert "(N_b + 1) / 8" in smp.describe()


def test_int8_keys_only_on_the_split_path():
    assert bench.parse(["--k-format", "int8"]).k_format == "int8"
    assert bench.parse(["--k-format", "int8", "--decode-path", "split"]).decode_path == "split"
    for path in ("fused", "tc"):
        with pytest.raises(SystemExit):
            bench.parse(["--k-format", "int8", "--decode-path", path])
