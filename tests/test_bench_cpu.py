"""Host-side byte accounting of bench.py (CPU only): the algorithmic bytes of
a decode launch and the unique bytes when sequences share prefix blocks."""
import math

import bench
import workloads as W

BYTES = bench.BYTES_PER_TOKEN_HEAD


def test_bytes_per_token_head():
    # two 128-byte code rows (K and V) and two fp32 scales per (token, KV head)
    assert BYTES == 2 * 128 + 2 * 4 == 264


def test_algorithmic_bytes_closed_form():
    w = W.make_workload("acct", 4242, [17, 300, 1], 8, 2)
    ab = bench.algorithmic_bytes(w)
    assert ab["kv"] == (17 + 300 + 1) * 2 * BYTES
    assert ab["q"] == ab["out"] == 3 * 8 * 128 * 2
    assert ab["tables"] == (2 + 19 + 1) * 4
    assert ab["total"] == ab["kv"] + ab["q"] + ab["out"] + ab["tables"]


def test_unique_bytes_without_sharing_equal_logical():
    w = W.make_workload("acct", 4243, [16, 33, 500], 16, 4)
    assert bench.unique_kv_bytes(w) == bench.algorithmic_bytes(w)["kv"]


def test_unique_bytes_with_shared_prefix():
    # 2 groups of 3 sequences share a 64-token prefix; one private sequence
    lens = [64 + 10, 64 + 40, 64 + 1, 64 + 17, 64 + 16, 64 + 33, 90]
    grp = [0, 0, 0, 1, 1, 1, -1]
    w = W.make_workload("acct", 4244, lens, 8, 2, prefix_group=grp, prefix_len=64)
    unique_tokens = 2 * 64 + sum(t - 64 for t, g in zip(lens, grp) if g >= 0) + 90
    assert bench.unique_kv_bytes(w) == unique_tokens * 2 * BYTES
    assert bench.algorithmic_bytes(w)["kv"] == sum(lens) * 2 * BYTES
    # the shared blocks really are the same physical blocks
    for g0 in (0, 3):
        for b in (g0 + 1, g0 + 2):
            assert list(w.block_tables[b, :4]) == list(w.block_tables[g0, :4])


def test_prefix_shared_workload_unique_share():
    w = W.prefix_shared_70b()
    u = bench.unique_kv_bytes(w)
    kv = bench.algorithmic_bytes(w)["kv"]
    prefix = 6 * 4096 * w.num_kv_heads * BYTES
    suffix = sum(int(t) - 4096 for t in w.context_lens) * w.num_kv_heads * BYTES
    assert u == prefix + suffix
    assert math.isclose(kv / u, (8 * prefix + suffix) / (prefix + suffix))


def test_kivi_algorithmic_bytes_closed_form():
    # full pages move their 2176-byte record per KV head; the partial page's
    # rows are read from the bf16 tail (K and V, 256 B each)
    assert bench.KIVI_PAGE_BYTES == 2 * 512 + 2 * 512 + 2 * 64 == 2176
    w = W.make_workload("kacct", 4244, [17, 300, 1, 32], 8, 2)
    kb = bench.kivi_algorithmic_bytes(w)
    full = 1 + 18 + 0 + 2
    rows = 1 + 12 + 1 + 0
    assert kb["kv"] == (full * 2176 + rows * 2 * 256) * 2
    ab = bench.algorithmic_bytes(w)
    assert kb["total"] == kb["kv"] + ab["q"] + ab["out"] + ab["tables"]
    # the bench workload: 136 B per (token, KV head), every page full
    big = W.llama8b_b64_32k()
    assert bench.kivi_algorithmic_bytes(big)["kv"] == 64 * 32768 * 8 * 136


def test_traffic_records_follow_their_own_sources():
    # each launch's record is keyed to the sources it is built from
    dec = bench.decode_sources()
    kivi = bench.decode_sources(bench.KIVI_ROOTS)
    assert "kv8_decode.cu" in dec and "kv8_api.cu" in dec
    assert "kv8_kivi.cu" not in dec and "kv8_decode.cu" not in kivi
    assert "kv8_kivi.cu" in kivi and "kv8_merge.cuh" in kivi
    assert bench.kernel_source_hash() != bench.kernel_source_hash(bench.KIVI_ROOTS)


def test_kivi_cpu_baseline_runs_the_oracle():
    w = W.make_workload("kcpu", 4245, [40, 17, 1, 0], 8, 2)
    sec, desc = bench.oracle_kivi_sample_seconds(w, [0, 1, 2, 3], threads=2)
    assert sec > 0 and "4 sequences" in desc and "2 threads" in desc
    sec1, desc1 = bench.oracle_kivi_sample_seconds(w, [1], threads=8)
    assert sec1 > 0 and "1 thread" in desc1


def test_int4_cpu_baseline_runs_the_oracle():
    w = W.make_workload("i4cpu", 4246, [40, 17, 1], 8, 2)
    sec, desc = bench.oracle_int4_sample_seconds(w, [0, 1, 2], threads=3)
    assert sec > 0 and "3 sequences" in desc and "3 threads" in desc
