"""Host-side pieces of bench.py that need no GPU: the measured-traffic lookup must
only report an ncu figure whose recorded source hash matches the kernel source as
it is now (a stale figure is reported as null)."""
import hashlib

import bench


def _profile(tmp_path, kernel_src: bytes, recorded: bytes, traffic="123.5e6"):
    csrc = tmp_path / "csrc"
    prof = tmp_path / "profiles"
    csrc.mkdir()
    prof.mkdir()
    (csrc / "k.cu").write_bytes(kernel_src)
    (prof / "k_w.md").write_text(f"# k on w\nsource_sha256: {hashlib.sha256(recorded).hexdigest()}\n"
                                 f"traffic_bytes_per_launch: {traffic}\n")
    return str(csrc), str(prof)


def test_traffic_is_reported_for_the_profiled_source(tmp_path, monkeypatch):
    csrc, prof = _profile(tmp_path, b"kernel v2", b"kernel v2")
    monkeypatch.setattr(bench, "CSRC", csrc)
    monkeypatch.setattr(bench, "PROFILES", prof)
    assert bench.traffic_from_profile("k.cu", "w") == 123.5e6


def test_traffic_is_null_once_the_kernel_changed(tmp_path, monkeypatch):
    csrc, prof = _profile(tmp_path, b"kernel v3", b"kernel v2")
    monkeypatch.setattr(bench, "CSRC", csrc)
    monkeypatch.setattr(bench, "PROFILES", prof)
    assert bench.traffic_from_profile("k.cu", "w") is None


def test_traffic_is_null_without_a_profile(tmp_path, monkeypatch):
    csrc, prof = _profile(tmp_path, b"kernel", b"kernel")
    monkeypatch.setattr(bench, "CSRC", csrc)
    monkeypatch.setattr(bench, "PROFILES", prof)
    assert bench.traffic_from_profile("k.cu", "other-workload") is None


def test_committed_profiles_name_their_source_and_traffic():
    """Every summary bench.py reads records a source hash and a per-launch traffic figure."""
    import os
    import re
    for name in os.listdir(bench.PROFILES):
        if name.startswith("launches_"):
            continue
        txt = open(os.path.join(bench.PROFILES, name)).read()
        assert re.search(r"source_sha256:\s*[0-9a-f]{64}", txt), name
        assert re.search(r"traffic_bytes_per_launch:\s*[0-9.eE+]+", txt), name
