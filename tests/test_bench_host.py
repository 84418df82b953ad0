"""Host-side pieces of bench.py that need no GPU: the kernel-source hash that ties recorded ncu traffic to the
code it was captured on, and the per-call launch count."""
import os

import bench
import synth


def test_strip_comments_keeps_code_and_literals():
    src = ('asm volatile("mbarrier.try_wait // kept-1");  // gone-1\n'
           "/* gone-2\n   gone-3 */ int x = '/';\n\n   \n"
           'const char *s = "a \\" quote /* kept */";\n')
    out = bench.strip_comments(src)
    assert "gone" not in out
    assert '"mbarrier.try_wait // kept-1"' in out
    assert '"a \\" quote /* kept */"' in out and "int x = '/';" in out
    assert "\n\n" not in out  # blank lines dropped


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    f = tmp_path / "k.cuh"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["k.cuh"])
    f.write_text("int a = 1;  // one\n")
    h1 = bench.kernel_source_hash()
    f.write_text("// header\nint a = 1;  /* still one */\n\n")
    assert bench.kernel_source_hash() == h1
    f.write_text("int a = 2;\n")
    assert bench.kernel_source_hash() != h1


def test_recorded_traffic_is_used_only_for_the_captured_code(tmp_path, monkeypatch):
    """A traffic record counts while its hash matches the kernel sources' code, and reads as null after that."""
    import json

    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as fh:
        records = json.load(fh)
    for rec in records.values():  # well formed: a 16-hex-digit hash and a positive byte count
        assert len(rec["kernel_hash"]) == 16 and int(rec["kernel_hash"], 16) >= 0 and rec["dram_bytes_per_launch"] > 0
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cuh").write_text("int a = 1;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["k.cuh"])
    rec = {"2": {"kernel_hash": bench.kernel_source_hash(), "dram_bytes_per_launch": 123, "source": "test"}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic(2) == 123
    assert bench.recorded_traffic(5) is None
    (tmp_path / "k.cuh").write_text("int a = 2;\n")
    assert bench.recorded_traffic(2) is None


def test_launches_per_call():
    dense = synth.make_dense(128, 256, 512)
    long_k = synth.make_dense(128, 256, 2176)
    nn = synth.make_contiguous_nn([129], 256, 256)
    assert bench.launches_per_call(dense) == 1  # a short call: the promotion GEMM alone
    assert bench.launches_per_call(long_k) == 2  # scale pre-pass + GEMM
    assert bench.launches_per_call(nn) == 2  # B read in place by the swapped-operand tiles
    assert bench.launches_per_call(nn, promotion=True) == 2  # transpose + the promotion GEMM
    assert bench.launches_per_call(dense, promotion=True) == 1  # the promotion GEMM has no pre-pass
