"""Host-side pieces of the benchmark's measurement contract (no GPU).

- The algorithmic bytes per element of each quantiser call kind follow from the
  format's storage cost: 4-bit codes plus one E4M3 byte per 16 elements (0.5625
  bytes per element, the format of aisight.pl, "Architektura NVFP4 kontra
  ograniczenia mikroskalowania", and the ~3.6x fewer bits than BF16 of
  aibuzzwire.news, Thinking Machines "End-to-End 4-Bit Training" article, section
  "Drei Formate, ein Trainingslauf"), and bf16 reads of 2 bytes per pass; MXFP4
  has one E8M0 byte per 32 elements.
- The DRAM traffic the bench reports comes from a committed ncu record, and only
  while that record was taken on the current GEMM source: a kernel change without
  a new capture must read as "no traffic", never as the old figure.
"""
import hashlib
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_quantiser_byte_counts():
    nvfp4_write = 0.5 + 1.0 / 16
    assert bench.quant_bytes_per_elem(None) == 2 + 2 + nvfp4_write          # amax pass + quantise pass
    assert bench.quant_bytes_per_elem(True) == 2 + nvfp4_write              # amax supplied: one read
    assert bench.quant_bytes_per_elem("amax") == 2                          # the amax pass alone
    assert bench.quant_bytes_per_elem("dual") == 2 + 2 + 2 * nvfp4_write    # both orientations from one read
    assert bench.MX_BYTES == 2 + 0.5 + 1.0 / 32
    assert abs(16 / (8 * nvfp4_write) - 3.56) < 0.01                        # bits vs bf16: the pages' ~3.6x


def test_step_flops():
    # six GEMMs of 2 * tokens * hidden * ffn each: Fprop, Dgrad, Wgrad of both projections
    assert bench.GEMM_FLOPS == 6 * 2 * 8192 * 5120 * 20480


def test_traffic_record_tracks_gemm_source():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["gemm_nvfp4_kernel"]
    src = os.path.join(ROOT, "nvfp4_bit_precision_quantize_b200", "csrc", rec["source"])
    with open(src, "rb") as f:
        current = hashlib.sha256(f.read()).hexdigest()[:16]
    got = bench.traffic_record("gemm_nvfp4_kernel")
    if current == rec["sha256_16"]:
        assert got is not None and got["bytes_per_launch"] == rec["read_bytes"] + rec["write_bytes"]
        assert os.path.exists(os.path.join(ROOT, rec["capture"]))
    else:
        assert got is None


def test_traffic_record_rejects_other_sources(tmp_path, monkeypatch):
    # a record whose hash does not match the source it names is ignored
    prof = tmp_path / "profiles"
    prof.mkdir()
    csrc = tmp_path / "nvfp4_bit_precision_quantize_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_bytes(b"kernel source v2\n")
    old = hashlib.sha256(b"kernel source v1\n").hexdigest()[:16]
    (prof / "traffic.json").write_text(json.dumps({"k": {"source": "k.cu", "sha256_16": old, "bytes_per_launch": 1}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k") is None
    new = hashlib.sha256(b"kernel source v2\n").hexdigest()[:16]
    (prof / "traffic.json").write_text(json.dumps({"k": {"source": "k.cu", "sha256_16": new, "bytes_per_launch": 1}}))
    assert bench.traffic_record("k")["bytes_per_launch"] == 1
