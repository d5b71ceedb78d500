"""Host-side checks of bench.py helpers (no GPU): the kernel-source digest that
keys the committed DRAM-traffic record ignores comments, and the traffic the
bench reports is the record's exactly when the record was taken of the
current attention kernel source (otherwise null)."""
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
