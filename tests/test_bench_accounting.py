"""The bench's per-launch accounting (host logic, no GPU): every traced
launch of a step gets the label of the work it does, and each label its
own algorithmic bytes or flops, so that a kernel's achieved rate divides
only its own launches' bytes by their own durations."""

import importlib.util
import os

from fp4_kv_cache_mxfp4_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)

Q_, S_, T_, A_, M_ = ("quantize_kv_fp4_kernel", "index_scan_kernel", "topk_select_kernel", "sparse_attn_tc_kernel",
                      "sparse_attn_combine_kernel")


def test_decoder_group_labels_and_bytes():
    wl = workloads.WORKLOADS[2]                     # Full, Reindex, Reindex, Reuse
    names = [Q_, S_, T_, A_, M_, S_, T_, A_, M_, S_, T_, A_, M_, A_, M_]
    labels = bench.label_launches(wl, names)
    assert labels == [
            "quantize", "scan", "topk", "attention", "attention_merge", "scan", "topk", "attention",
            "attention_merge", "scan", "topk", "attention", "attention_merge", "attention", "attention_merge"]
    assert bench.label_work(wl, "scan") == ("hbm", 4 * (131072 * 256 + 131072 * 4 + 32 * 128 * 2 + 32 * 4), "B")
    assert bench.label_work(wl, "scan")[1] == 136348160
    att = 4 * (512 * 4 + 512 * 288 + 128 * 1024 + 2 * 64 * 512 * 2)
    assert bench.label_work(wl, "attention") == ("hbm", att, "B")
    # the same launches without the merge kernel label the same way
    names2 = [Q_, S_, T_, A_, S_, T_, A_, S_, T_, A_, A_]
    assert bench.label_launches(wl, names2) == ["quantize", "scan", "topk", "attention", "scan", "topk", "attention",
                                                "scan", "topk", "attention", "attention"]


def test_hsi_labels_split_full_scan_from_pool_rescore():
    """At 1M entries the Full scan and a pool re-score differ by 64x in
    bytes; they must not share one average."""
    wl = workloads.WORKLOADS[3]
    names = [Q_, S_, T_, T_, A_, S_, T_, A_, S_, T_, A_, S_, T_, A_]
    labels = bench.label_launches(wl, names)
    assert labels == ["quantize", "scan", "topk", "topk_blocks", "attention", "scan_pool", "topk_pool", "attention",
                      "scan_pool", "topk_pool", "attention", "scan_pool", "topk_pool", "attention"]
    full = bench.label_work(wl, "scan")[1]
    pool = bench.label_work(wl, "scan_pool")[1]
    assert full == 2 * (1048576 * 260 + 32 * 128 * 2 + 32 * 4)
    assert pool == 2 * (2048 * 4 + 16384 * 260 + 32 * 128 * 2 + 32 * 4)
    assert 60 < full / pool < 66
    assert bench.label_work(wl, "topk_blocks")[1] == 2 * (131072 * 4 + 2048 * 4)


def test_prefill_scan_is_counted_in_flops():
    wl = workloads.WORKLOADS[4]
    labels = bench.label_launches(wl, [Q_, S_, T_, A_])
    assert labels == ["quantize", "scan_prefill", "topk", "attention"]
    bound, flops, unit = bench.label_work(wl, "scan_prefill")
    assert bound == "tensor" and unit == "flop"
    assert flops == 8192 * sum(wl.n_vis)


def test_step_bytes_count_each_mode_once():
    wl = workloads.WORKLOADS[3]
    want = (bench.scan_algorithmic_bytes(wl) + 3 * bench.pool_scan_algorithmic_bytes(wl)
            + bench.quantize_algorithmic_bytes(wl) + 4 * bench.attention_algorithmic_bytes(wl))
    assert bench.step_algorithmic_bytes(wl) == want


def test_both_arms_print_the_same_config():
    wl = workloads.WORKLOADS[2]
    c = bench.bench_config(wl, 1)
    assert c["workload"] == "group4_decode_ctx128k_b4" and c["N_entries"] == 131072 and c["r"] == 1
    assert c["layers"] == "full,reindex,reindex,reuse" and c["kv_cache"].startswith("FP4")


def test_scan_kernel_names():
    """One query per MMA group (decode rows, pool re-scores) runs the
    transposed scan; several queries per group the other one."""
    assert bench.scan_kernel_name(workloads.WORKLOADS[2], "scan") == "index_scan_t_kernel"
    assert bench.scan_kernel_name(workloads.WORKLOADS[3], "scan_pool") == "index_scan_t_kernel"
    assert bench.scan_kernel_name(workloads.WORKLOADS[4], "scan_prefill") == "index_scan_kernel"
    assert workloads.WORKLOADS[4].Q > 1


def test_source_digest_ignores_comments_not_code():
    """The recorded scan traffic stays valid across comment edits and is
    dropped by any change of code."""
    src = 'int f(int a) {  // the query\'s tile\n  /* two\n lines */ return a + 1; }\nconst char* s = "//x";\n'
    base = bench.code_tokens(src)
    assert base == 'int f(int a) { return a + 1; } const char* s = "//x";'
    assert bench.code_tokens(src.replace("the query's tile", "another comment")) == base
    assert bench.code_tokens(src.replace("  return", "\n\n    return")) == base
    assert bench.code_tokens(src.replace("a + 1", "a + 2")) != base
    assert bench.code_tokens(src.replace('"//x"', '"//y"')) != base
    assert len(bench.kernel_source_sha()) == 16
