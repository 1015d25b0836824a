"""bench.py's reporting of the forward kernel's ncu DRAM traffic: the recorded
number is used only while it was taken on the current kernel source."""
import os

import bench


def _tree(tmp_path, sources, traffic_text):
    csrc = tmp_path / "io_aware_exact_31_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, body in sources.items():
        (csrc / name).write_bytes(body)
    prof = tmp_path / "profiles"
    prof.mkdir()
    if traffic_text is not None:
        (prof / "fwd_traffic.txt").write_text(traffic_text)
    return str(tmp_path)


def test_traffic_follows_the_kernel_source_hash(tmp_path, monkeypatch):
    sources = {"fa_fwd.cuh": b"kernel", "sm100.cuh": b"helpers", "philox.cuh": b"rng"}
    root = _tree(tmp_path, sources, None)
    monkeypatch.setattr(bench, "ROOT", root)
    h = bench.kernel_source_hash()
    assert len(h) == 12

    prof = os.path.join(root, "profiles", "fwd_traffic.txt")
    with open(prof, "w") as f:
        f.write(f"# comment = ignored\nkernel_source_sha1_12={h}\ndram_bytes_per_launch=1234\n")
    assert bench.recorded_traffic() == 1234

    # Any change to a hashed source makes the recorded number stale.
    with open(os.path.join(root, "io_aware_exact_31_b200", "csrc", "philox.cuh"), "ab") as f:
        f.write(b" ")
    assert bench.kernel_source_hash() != h
    assert bench.recorded_traffic() is None


def test_traffic_missing_or_malformed_is_none(tmp_path, monkeypatch):
    sources = {"fa_fwd.cuh": b"a", "sm100.cuh": b"b", "philox.cuh": b"c"}
    root = _tree(tmp_path, sources, None)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.recorded_traffic() is None
    with open(os.path.join(root, "profiles", "fwd_traffic.txt"), "w") as f:
        f.write(f"kernel_source_sha1_12={bench.kernel_source_hash()}\ndram_bytes_per_launch=x\n")
    assert bench.recorded_traffic() is None


def test_committed_traffic_record_is_well_formed():
    """The committed record names a 12-hex-digit source hash and a byte count
    of the right order for the 4x16x4096x128 forward (inputs + output)."""
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles",
                        "fwd_traffic.txt")
    d = {}
    for line in open(path):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.strip().split("=", 1)
            d[k] = v
    assert len(d["kernel_source_sha1_12"]) == 12
    int(d["kernel_source_sha1_12"], 16)
    assert 150e6 < int(d["dram_bytes_per_launch"]) < 400e6
