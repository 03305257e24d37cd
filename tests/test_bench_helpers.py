"""Host-side helpers of bench.py (CPU): the recorded DRAM traffic is reported only for the kernel
source it was captured on, a figure may carry its own source hash, and the source hash ignores
comments and blank lines but not code."""
import bench


def _write(tmp_path, text):
    p = tmp_path / "traffic.txt"
    p.write_text(text)
    return str(p)


def test_traffic_needs_the_current_kernel_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, (
        "# comment\nkernel_source_sha256_16 = %s\nbytes_per_launch_full = 123\n" % h)))
    assert bench.recorded_traffic("full") == 123.0
    assert bench.recorded_traffic("micro") is None          # no figure for it
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, (
        "kernel_source_sha256_16 = 0000000000000000\nbytes_per_launch_full = 123\n")))
    assert bench.recorded_traffic("full") is None            # taken on another kernel


def test_a_figure_can_carry_its_own_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    h8 = bench.kernel_source_hash(bench.KERNEL_SOURCES_INT8)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, (
        "kernel_source_sha256_16 = %s\n"
        "kernel_source_sha256_16_full_int8 = 0123456789abcdef\n"
        "bytes_per_launch_full = 10\nbytes_per_launch_full_int8 = 20\n" % h)))
    assert bench.recorded_traffic("full") == 10.0
    assert bench.recorded_traffic("full_int8") is None       # older capture
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, (
        "kernel_source_sha256_16 = 0123456789abcdef\n"
        "kernel_source_sha256_16_full_int8 = %s\n"
        "bytes_per_launch_full = 10\nbytes_per_launch_full_int8 = 20\n" % h8)))
    assert bench.recorded_traffic("full") is None
    assert bench.recorded_traffic("full_int8") == 20.0


def test_each_kernel_has_its_own_source_hash(tmp_path, monkeypatch):
    # a change to the pair kernel's source leaves the INT8 kernel's figures valid, and the
    # reverse; a source both kernels read invalidates both
    src = tmp_path / "csrc"
    src.mkdir()
    for f in set(bench.KERNEL_SOURCES) | set(bench.KERNEL_SOURCES_INT8):
        (src / f).write_text("int %s = 1;\n" % f.split(".")[0])
    monkeypatch.setattr(bench, "CSRC", str(src))
    h, h8 = bench.kernel_source_hash(), bench.kernel_source_hash(bench.KERNEL_SOURCES_INT8)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _write(tmp_path, (
        "kernel_source_sha256_16 = %s\nkernel_source_sha256_16_int8 = %s\n"
        "bytes_per_launch_full = 10\nbytes_per_launch_full_int8 = 20\n" % (h, h8))))
    assert bench.recorded_traffic("full") == 10.0 and bench.recorded_traffic("full_int8") == 20.0
    (src / "attn_pair.cuh").write_text("int changed = 2;\n")
    assert bench.recorded_traffic("full") is None and bench.recorded_traffic("full_int8") == 20.0
    (src / "attn_pair.cuh").write_text("int attn_pair = 1;\n")
    (src / "quant_int8.cuh").write_text("int changed = 2;\n")
    assert bench.recorded_traffic("full") == 10.0 and bench.recorded_traffic("full_int8") is None
    (src / "quant_int8.cuh").write_text("int quant_int8 = 1;\n")
    (src / "tara_common.cuh").write_text("int changed = 2;\n")
    assert bench.recorded_traffic("full") is None and bench.recorded_traffic("full_int8") is None


def test_missing_file_reports_nothing(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.txt"))
    assert bench.recorded_traffic("full") is None


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    src = tmp_path / "csrc"
    src.mkdir()
    for f in bench.KERNEL_SOURCES:
        (src / f).write_text("int a = 1;  // one\n\nint b = 2;\n")
    monkeypatch.setattr(bench, "CSRC", str(src))
    h0 = bench.kernel_source_hash()
    (src / bench.KERNEL_SOURCES[0]).write_text("// a new comment\nint a = 1;\n   \nint b = 2;   // two\n")
    assert bench.kernel_source_hash() == h0
    (src / bench.KERNEL_SOURCES[0]).write_text("int a = 1;\nint b = 3;\n")
    assert bench.kernel_source_hash() != h0



def test_clock_normalised_fraction():
    peaks = {"clocks_under_load": {"sm_mhz_median": 1300.0}}
    # a kernel at twice the peak's clock: the per-clock fraction is half the plain one
    r = bench.clock_normalised(1000.0, 1400.0, 2600.0, peaks)
    assert abs(r["frac_at_kernel_clock"] - 1000.0 / 2800.0) < 1e-12
    assert r["kernel_sm_mhz_median"] == 2600.0 and r["peak_sm_mhz_median"] == 1300.0
    # at the peak's own clock both fractions agree
    assert abs(bench.clock_normalised(700.0, 1400.0, 1300.0, peaks)["frac_at_kernel_clock"] - 0.5) < 1e-12
    # an unknown clock gives no figure rather than a guess
    assert bench.clock_normalised(1.0, 2.0, None, peaks)["frac_at_kernel_clock"] is None
    assert bench.clock_normalised(1.0, 2.0, 1500.0, {})["frac_at_kernel_clock"] is None
