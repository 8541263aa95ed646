"""Host logic of bench.py that needs no GPU: the traffic record is reported only while the
streaming kernel's code (comments aside) is the code its counters were taken on."""
import hashlib
import json

import bench


def test_kernel_code_ignores_comments_and_blank_lines():
    a = "int x = 1;  // the count\n\n// a whole-line note\nint y = 2;\n"
    b = "int x = 1;\n// another note\n\nint y = 2;  // changed comment\n"
    assert bench.kernel_code(a) == bench.kernel_code(b) == "int x = 1;\nint y = 2;"
    assert bench.kernel_code(a) != bench.kernel_code(a.replace("2;", "3;"))


def _tree(tmp_path, src: str, key_src: str, traffic: int):
    csrc = tmp_path / "draft_token_verification_spec_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "stream.cuh").write_text(src)
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(bench.kernel_code(key_src).encode()).hexdigest()[:16]
    rec = {"stream_cuh_sha256_16": sha, "traffic": {"w": traffic}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))


def test_traffic_reported_while_the_code_matches(tmp_path, monkeypatch):
    src = "__global__ void k() {}  // v1\n"
    _tree(tmp_path, src, src.replace("v1", "comment edited"), 12345)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_profile_traffic("w") == 12345
    assert bench.read_profile_traffic("other workload") is None


def test_traffic_null_once_the_code_changes(tmp_path, monkeypatch):
    _tree(tmp_path, "__global__ void k() { int a; }\n", "__global__ void k() {}\n", 12345)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_profile_traffic("w") is None


def test_traffic_null_without_a_record(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_profile_traffic("w") is None
