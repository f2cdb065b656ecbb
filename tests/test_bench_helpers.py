"""Host-side helpers of bench.py that decide whether a committed DRAM-traffic
record still describes the kernel being measured."""
import json
import os

import bench

SRC = ('// leading remark\n__device__ int f(int x) {  /* block\n comment */\n'
       '  asm volatile("mov.u32 %0, %1; // not a comment" : "=r"(x) : "r"(x));\n'
       '  return x + 1;  // trailing\n}\n')


def test_strip_comments_keeps_code_and_string_literals():
    out = bench.strip_comments(SRC)
    assert "leading remark" not in out and "block" not in out and "trailing" not in out
    assert '"mov.u32 %0, %1; // not a comment"' in out
    assert "return x + 1;" in out
    # escaped quotes inside a literal do not end it
    assert bench.strip_comments('s = "a \\" // b"; // c') == 's = "a \\" // b";'


def test_comment_and_layout_edits_keep_the_code_identity():
    edited = SRC.replace("// leading remark", "// another remark").replace("  return", "\n\n    return")
    assert bench.strip_comments(edited) == bench.strip_comments(SRC)
    changed = SRC.replace("x + 1", "x + 2")
    assert bench.strip_comments(changed) != bench.strip_comments(SRC)


def test_workloads_map_to_their_kernel():
    assert bench.uses_prefill_kernel("chunked_prefill")        # 512 new tokens x G 4 >= 128 rows
    for w in ("llama3_8b", "llama3_70b_32k", "prefix_shared", "quant_mha", "spec_verify", "tiny"):
        assert not bench.uses_prefill_kernel(w)


def test_traffic_records_are_well_formed():
    path = os.path.join(bench.ROOT, "profiles", "kernel_traffic.json")
    with open(path) as f:
        records = json.load(f)
    for key, rec in records.items():
        assert rec["dram_bytes_per_call"] > 0
        assert len(rec["source_hash"]) == 16
        assert rec["capture"].startswith("ncu ") and "--clock-control none" in rec["capture"]
        if rec["alg_bytes_per_call"] is None:
            # an L2 record, reported as captured (never scaled)
            assert 0 < rec["l2_sector_hit_pct"] <= 100
            assert bench.recorded_traffic(key, None, 10 ** 9) is None
            continue
        assert rec["alg_bytes_per_call"] > 0
        # a record scales with the algorithmic bytes of the call it is used for
        if rec["source_hash"] == bench.kernel_source_hash(
                bench.PREFILL_SOURCES if key == "chunked_prefill" else bench.DECODE_SOURCES):
            wl, cache = ("quant_mha", key.split("quant_mha_")[1]) if key.startswith("quant_mha_") else (key, None)
            got = bench.recorded_traffic(wl, cache, 2 * rec["alg_bytes_per_call"])
            assert abs(got - 2 * rec["dram_bytes_per_call"]) <= 2
