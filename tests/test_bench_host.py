"""Host-side logic of bench.py that needs no GPU: band pair counts and the lookup of a kernel's
measured DRAM traffic from its committed ncu summary."""
import hashlib
import os

import bench


def test_band_pairs_matches_brute_force():
    for T in (1, 5, 130):
        for W in (1, 3, 64, 129, 130, 500):
            brute = sum(1 for i in range(T) for j in range(T) if i - W < j <= i)
            assert bench.band_pairs(T, W) == brute, (T, W)


def _fake_root(tmp_path, line):
    csrc = tmp_path / "causal_sliding_window_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cuh").write_text("kernel a\n")
    (csrc / "b.cuh").write_text("helpers b\n")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "swa_bwd_dkdv_kernel_d24shape_b8.md").write_text("# summary\n\n" + line + "\n")
    return tmp_path


def test_measured_traffic_scales_and_averages(tmp_path, monkeypatch):
    sha = hashlib.sha256(b"kernel a\nhelpers b\n").hexdigest()
    root = _fake_root(tmp_path, f"traffic_bytes: W=2048 400; W=512 200; batch 8; source_sha256 {sha} (a.cuh + b.cuh)")
    monkeypatch.setattr(bench, "ROOT", str(root))
    # batch 32 = 4x the captured batch; the step has three W=512 launches and one W=2048 launch
    assert bench.measured_traffic("swa_bwd_dkdv_kernel<128>", [512, 512, 512, 2048], 32) == (3 * 200 + 400) / 4 * 4
    assert bench.measured_traffic("swa_bwd_dkdv_kernel<128>", [1024], 32) is None      # window not captured
    assert bench.measured_traffic("no_such_kernel", [512], 32) is None


def test_measured_traffic_is_null_once_the_sources_change(tmp_path, monkeypatch):
    stale = hashlib.sha256(b"an older kernel\n").hexdigest()
    root = _fake_root(tmp_path, f"traffic_bytes: W=512 200; batch 8; source_sha256 {stale} (a.cuh + b.cuh)")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.measured_traffic("swa_bwd_dkdv_kernel<128>", [512], 32) is None


def test_committed_summaries_parse():
    for kernel in bench.PROFILE_FOR_KERNEL:
        path = os.path.join(bench.ROOT, "profiles", bench.PROFILE_FOR_KERNEL[kernel])
        assert os.path.exists(path), path
        assert "traffic_bytes: " in open(path).read(), path
