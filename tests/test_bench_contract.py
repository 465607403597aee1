"""bench.py's recorded DRAM traffic of the S2 GEMM applies only to the kernel
sources it was measured on: the bench reports it while every listed source
still has its recorded SHA-256, and null as soon as one differs (CPU only)."""
import hashlib

import bench


def _record_for(root, files):
    srcs = {}
    for rel, text in files.items():
        path = root / rel
        path.parent.mkdir(parents=True, exist_ok=True)
        path.write_bytes(text)
        srcs[rel] = hashlib.sha256(text).hexdigest()
    return {"bytes": 12345, "sources": srcs}


def test_traffic_reported_while_sources_match(tmp_path, monkeypatch):
    rec = _record_for(tmp_path, {"csrc/k.cu": b"kernel", "csrc/h.cuh": b"header"})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", rec)
    assert bench._gemm_traffic() == 12345


def test_traffic_dropped_when_a_source_changes(tmp_path, monkeypatch):
    rec = _record_for(tmp_path, {"csrc/k.cu": b"kernel", "csrc/h.cuh": b"header"})
    (tmp_path / "csrc/h.cuh").write_bytes(b"header, edited")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", rec)
    assert bench._gemm_traffic() is None


def test_traffic_dropped_when_a_source_is_missing(tmp_path, monkeypatch):
    rec = _record_for(tmp_path, {"csrc/k.cu": b"kernel"})
    rec["sources"]["csrc/gone.cu"] = "0" * 64
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", rec)
    assert bench._gemm_traffic() is None


def test_recorded_sources_are_the_s2_kernel_files():
    srcs = bench.GEMM_TRAFFIC["sources"]
    assert "bit_w4a4_diffusion_b200/csrc/gemm_nvfp4_pair.cu" in srcs
    assert all(len(d) == 64 for d in srcs.values())
