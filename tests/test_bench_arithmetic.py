"""bench.py's roofline arithmetic (CPU): the counted FLOPs and algorithmic
bytes per workload against the figures the workload definitions fix, written
out here term by term, and the traffic registry's gate (a DRAM figure is
reported only while the code it was captured on is unchanged)."""
import hashlib
import json

import pytest

import bench

STATE = 48 * 128 * 128 * 4          # one sequence's fp32 state, 48 value heads
PER_TOKEN = (2 * 16 * 128 * 2       # q, k (bf16)
             + 3 * 48 * 128 * 2     # v, g, y (bf16)
             + 2 * 48 * 4)          # log alpha, beta (fp32)


def test_prefill_per_token_bytes_are_45440():
    assert PER_TOKEN == 45_440
    # no epilogue: g is not read, norm_w neither
    assert bench.prefill_bytes(1, 0, epilogue=False) == PER_TOKEN - 48 * 128 * 2


@pytest.mark.parametrize("T,n_seq,init,expected", [
    (4096, 1, False, 189_268_480),                    # model shape, zero initial state
    (4096, 1, True, 45_440 * 4096 + 2 * STATE + 512),  # ~192.4 MB with a state read
    (262_144, 1, True, 45_440 * 262_144 + 2 * STATE + 512),  # ~11.92 GB
])
def test_prefill_bytes(T, n_seq, init, expected):
    got = bench.prefill_bytes(T, n_seq, init_state=init)
    assert got == expected
    assert got == PER_TOKEN * T + STATE * n_seq * (2 if init else 1) + 128 * 4


def test_prefill_bytes_headline_values():
    assert round(bench.prefill_bytes(4096, 1) / 1e6, 1) == 192.4
    assert round(bench.prefill_bytes(262_144, 1) / 1e9, 2) == 11.92


def test_counted_flops_per_token():
    d, C = 128, 64
    per_v = 6 * d * d + 6 * C * d + C * C / 3
    per_qk = 4 * C * d
    assert bench.flops_per_token() == pytest.approx(48 * per_v + 16 * per_qk, rel=0, abs=1e-6)
    assert round(bench.flops_per_token() / 1e6, 2) == 7.67
    assert round(bench.flops_per_token() * 4096 / 1e9, 1) == 31.4


def test_decode_bytes():
    per_seq = 2 * STATE + 2 * 16 * 128 * 2 + 2 * 48 * 128 * 2 + 48 * 8
    assert bench.decode_bytes(256) == 256 * per_seq == 1_619_099_648


def test_backward_bytes_and_flops():
    per_tok = (2 * 16 * 128 * 2 + 3 * 48 * 128 * 2 + 48 * 8     # q, k, v, g, dy, gates in
               + 2 * 16 * 128 * 4 + 2 * 48 * 128 * 4 + 48 * 8)  # dq, dk, dv, dg, dgates out
    assert per_tok == 111_360
    assert bench.bwd_bytes(4096, 1) == per_tok * 4096 + 2 * STATE + 512
    assert round(bench.bwd_bytes(4096, 1) / 1e6, 1) == 462.4
    assert round(bench.bwd_flops_per_token() / 1e6, 1) == 25.0


def test_whole_job_rate_counts_every_rank():
    assert bench.whole_job_rate(4096, 1, 1.0) == pytest.approx(4.096e6)
    assert bench.whole_job_rate(4096, 8, 2.0) == pytest.approx(8 * 4096 / 2e-3)


def test_traffic_registry_gate(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    reg = {"k": {"source": "k.cu", "source_sha": sha, "bytes_per_launch": 1234}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(reg))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("k") == 1234.0
    assert bench.kernel_traffic("missing") is None
    src.write_text("kernel source, edited\n")   # changed since the capture: no figure
    assert bench.kernel_traffic("k") is None


def test_code_gate_ignores_comments_only(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text('// header\nint f(int x) { return x + 1; }  // tail\n'
                   'const char* s = "// kept";\n/* block\n comment */ int g;\n')
    (tmp_path / "profiles").mkdir()
    reg = {"k": {"source": "k.cu", "source_sha": "0" * 16, "code_sha": bench.code_sha(str(src)),
                 "bytes_per_launch": 99}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(reg))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("k") == 99.0
    # reworded and reflowed comments, blank lines: the same code
    src.write_text('// a new header,\n// two lines long\n\nint f(int x) { return x + 1; }\n'
                   'const char* s = "// kept";\n/* other */ int g;\n')
    assert bench.kernel_traffic("k") == 99.0
    # a string literal is code, even when it looks like a comment
    src.write_text('int f(int x) { return x + 1; }\nconst char* s = "// edited";\nint g;\n')
    assert bench.kernel_traffic("k") is None
    # so is any other change
    src.write_text('int f(int x) { return x + 2; }\nconst char* s = "// kept";\nint g;\n')
    assert bench.kernel_traffic("k") is None


def test_registered_sources_exist():
    reg = json.load(open(bench.ROOT + "/profiles/traffic.json"))
    for key, entry in reg.items():
        assert entry["bytes_per_launch"] > 0, key
        with open(bench.ROOT + "/" + entry["source"], "rb"):
            pass
