"""Host-side checks of bench.py helpers (no GPU): the kernel-source digest that
keys the committed DRAM-traffic record ignores comments; the traffic the bench
reports is the record's exactly when the record was taken of the current
attention kernel source (otherwise null); and the clock record keeps the
median SM clock of the samples under load and every active throttle reason."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("_bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_digest_ignores_comments(tmp_path):
    b = _bench()
    a = tmp_path / "a.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f() {\n  return 1;  // one\n}\n/* block\n comment */\n")
    c.write_text("// header\nint f() {\n\n  return 1;\n}\n")
    assert b.kernel_source_digest(str(a)) == b.kernel_source_digest(str(c))
    c.write_text("int f() {\n  return 2;\n}\n")
    assert b.kernel_source_digest(str(a)) != b.kernel_source_digest(str(c))


def test_traffic_reported_only_for_the_captured_kernel():
    import json
    b = _bench()
    rec = json.load(open(os.path.join(ROOT, "profiles",
                                      "chunk_attn_pair_kernel_ctx128k_traffic.json")))
    src = os.path.join(ROOT, "block_sparse_chunked_b200", "csrc", "attn_pair.cu")
    same = b.kernel_source_digest(src) == rec["source_digest"]
    t = b.load_traffic()
    if same:
        assert t == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    else:
        assert t is None


def _smi(mhz, watts, power_cap="Not Active", hw="Not Active"):
    """One line of the bench's nvidia-smi query (csv, no header, no units)."""
    return f"0, {mhz}, 1965, {watts}, 0x0000000000000004, {hw}, Not Active, Not Active, {power_cap}"


def test_clock_record_takes_the_median_under_load():
    b = _bench()
    idle = [_smi(1965, 120.0)] * 6
    load = [_smi(1837, 410.0, "Active"), _smi(1845, 405.0), _smi(1830, 420.0)]
    r = b.ClockSampler.summarize(idle + load + ["", "garbage", "0, n/a, 1965, 1, x, a, b, c, d"])
    assert r["sm_mhz"] == 1837.0                    # idle samples at 1965 MHz do not count
    assert r["samples"] == 9 and r["samples_under_load"] == 3
    assert r["sm_max_mhz"] == 1965.0 and r["power_w_max"] == 420.0
    assert r["reasons"] == ["sw_power_cap"]         # "Not Active" is not "Active"


def test_clock_record_flat_power_and_reasons():
    b = _bench()
    flat = [_smi(1900, 300.0), _smi(1910, 305.0), _smi(1890, 310.0, hw="Active")]
    r = b.ClockSampler.summarize(flat)
    assert r["samples_under_load"] == 3 and r["sm_mhz"] == 1900.0   # range under 20 W: all
    assert r["reasons"] == ["hw_slowdown"]
    assert b.ClockSampler.summarize([])["reasons"] == ["no samples"]
