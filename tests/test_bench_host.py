"""Host-side logic of bench.py that needs no GPU: the digest that keeps the
stored ncu traffic figures tied to the kernels' code, and the decode
configuration both arms report."""
import bench


def test_digest_ignores_comments_but_not_code():
    src = "int a = 1;  // one\n/* block\n comment */\nint b = a;\n\n// trailing\n"
    assert bench.strip_comments(src) == "int a = 1;\nint b = a;"
    files = ("x.cu",)
    base = bench.source_digest(files, read=lambda f: src)
    assert bench.source_digest(files, read=lambda f: src.replace("// one", "// a new note")) == base
    assert bench.source_digest(files, read=lambda f: "/* header */\n" + src) == base
    assert bench.source_digest(files, read=lambda f: src.replace("a = 1", "a = 2")) != base


def test_stored_digests_cover_the_kernel_sources():
    for files, stored in ((bench.STACK_SOURCES, bench.STACK_TRAFFIC), (bench.PREFILL_SOURCES, bench.PREFILL_TRAFFIC)):
        assert len(stored["digest"]) == 16
        assert all(f.startswith("csrc/") for f in files)
        assert stored["dram_bytes"] > 0


def test_both_arms_report_one_decode_config():
    c = bench.decode_config(1, 1)
    assert c["layers"] == bench.N_LAYERS and c["global_batch"] == 1 and c["parallelism"] == "replicas1"
    assert "48 stacked MoE layers" in c["workload"] or str(bench.N_LAYERS) in c["workload"]
