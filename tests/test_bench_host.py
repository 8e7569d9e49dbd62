"""Host-side logic of bench.py (no GPU): the ncu-traffic lookup that fills
`roofline.traffic`, its invalidation when a kernel source changes, the
whole-job throughput arithmetic, the launch count of the timed regions and
the quantise ALU-roofline constants."""
import os
import shutil

import pytest

import bench


def _fields(name):
    text = open(os.path.join(bench.ROOT, "profiles", name)).read()
    return dict(ln.split(": ", 1) for ln in text.splitlines() if ": " in ln and ln.split(": ", 1)[0] in
                ("traffic_bytes_per_launch", "weights_per_launch", "source_sha256"))


@pytest.mark.parametrize("phase", sorted(bench.PROFILE_FILES))
def test_profile_summaries_carry_traffic_fields(phase):
    name, sources = bench.PROFILE_FILES[phase]
    f = _fields(name)
    assert int(f["traffic_bytes_per_launch"]) > 0
    assert int(f["weights_per_launch"]) > 0
    assert len(f["source_sha256"].strip()) == 16
    for src in sources:
        assert os.path.exists(os.path.join(bench.ROOT, "dequant_gemv_tq4_b200", "csrc", src))


def _mirror(tmp_path, phase, edit_source=False, edit_hash=None):
    """A copy of the profile and the sources it hashes, under tmp_path."""
    name, sources = bench.PROFILE_FILES[phase]
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "dequant_gemv_tq4_b200" / "csrc"
    csrc.mkdir(parents=True)
    shutil.copy(os.path.join(bench.ROOT, "profiles", name), tmp_path / "profiles" / name)
    for src in sources:
        shutil.copy(os.path.join(bench.ROOT, "dequant_gemv_tq4_b200", "csrc", src), csrc / src)
    if edit_source:
        with open(csrc / sources[-1], "a") as f:
            f.write("\n// changed\n")
    if edit_hash is not None:
        p = tmp_path / "profiles" / name
        p.write_text(p.read_text().replace(_fields(name)["source_sha256"], edit_hash))


def test_traffic_scales_with_weights_and_tracks_the_source(tmp_path, monkeypatch):
    phase = "gemv"
    name, _ = bench.PROFILE_FILES[phase]
    f = _fields(name)
    traffic, per = int(f["traffic_bytes_per_launch"]), int(f["weights_per_launch"])
    # a summary whose hash matches its sources scales in proportion to the weights
    good = tmp_path / "good"
    good.mkdir()
    _mirror(good, phase, edit_hash=None)
    import hashlib
    h = hashlib.sha256()
    for src in bench.PROFILE_FILES[phase][1]:
        h.update((good / "dequant_gemv_tq4_b200" / "csrc" / src).read_bytes())
    p = good / "profiles" / name
    p.write_text(p.read_text().replace(f["source_sha256"], h.hexdigest()[:16]))
    monkeypatch.setattr(bench, "ROOT", str(good))
    assert bench.profile_traffic(phase, per) == traffic
    assert bench.profile_traffic(phase, 2 * per) == 2 * traffic
    # a source edited after the capture invalidates the figure
    stale = tmp_path / "stale"
    stale.mkdir()
    _mirror(stale, phase, edit_source=True)
    monkeypatch.setattr(bench, "ROOT", str(stale))
    assert bench.profile_traffic(phase, per) is None


def test_job_throughput_is_all_ranks_over_the_slowest():
    assert bench.job_gbs(1_000_000_000, 1, 1000.0) == pytest.approx(1.0)
    assert bench.job_gbs(1_000_000_000, 4, 1000.0) == pytest.approx(4.0)
    assert bench.max_over_ranks([1.0, 2.0], 1) == [1.0, 2.0]


def test_timed_launch_count():
    """The Llama layer (7 matrices), 20 replays of 10 step / quantise /
    dequantise passes and of 32 GEMV passes."""
    got = bench.timed_launches(7, 20, 10, 32)
    assert got["step"] == 10 * 20 * 10  # 7 quantise + 1 dequantise + pre-rotation + product per step
    assert got["quantize"] == 7 * 200 and got["dequantize"] == 200
    assert got["gemv"] == 2 * 20 * 32 and got["gemv_single_matrix"] == 2 * 20 * 7
    assert got["total"] == sum(v for k, v in got.items() if k != "total") == 5160


def test_quantise_alu_operation_count():
    # per 32-element block: sign flip, five butterfly stages, half-block RMS
    # (squares, pairwise adds, scale / root / rounding per half), thresholds,
    # three compares and a sign test per element, one nibble insert each
    block = 32 + 5 * 32 + (32 + 2 * 15 + 2 * 3) + 2 * 7 + 4 * 32 + 32
    assert block == 434
    assert bench.QUANT_OPS_PER_WEIGHT == pytest.approx(block / 32)
    assert bench.LANES_PER_SM == 128


def test_cpu_sample_and_row_partitioned_oracle():
    """The CPU baseline's sample is the first 1/8 of each matrix's rows
    (at least 16), and the row-partitioned run applies the oracle to slices
    of whole 16-row tiles: it produces exactly the packed bytes of the
    single-threaded run."""
    import numpy as np

    assert bench.cpu_sample_rows(4096) == 512
    assert bench.cpu_sample_rows(40) == 16
    assert bench.cpu_sample_rows(4096, 100) == 100
    rng = np.random.default_rng(3)
    mats = [(rng.standard_normal((50, 96)).astype(np.float32) * 0.02, rng.standard_normal((1, 96))),
            (rng.standard_normal((33, 160)).astype(np.float32) * 0.02, rng.standard_normal((1, 160)))]
    one = bench.oracle_pass(mats, 1)
    three = bench.oracle_pass(mats, 3)
    assert one[3] == three[3] > 0
