"""Host-side arithmetic of bench.py: the byte model behind the roofline
numerator (config 1 figures worked out field by field), the whole-job rate,
rank seeding, the comment-blind source hash, and the CPU oracle leg."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.fixture(scope="module")
def bench():
    import bench as b
    return b


@pytest.fixture(scope="module")
def wl():
    from linear_attention_recurrent_lq_b200 import inputs as I
    return I.WORKLOADS["gdn_int8_b64h32"]


def test_decode_bytes_by_hand(bench, wl):
    # header 20 + meta 16 + qs 512 + sm 512 + compensators 4*4*128 = 2048 + codes 128*128
    # + inputs (q, k, v bf16: 3*256, beta and alpha 4 + 4) = 776; writes: out 512,
    # the new pair 1024, count and g 8
    reads = 20 + 16 + 512 + 512 + 2048 + 16384 + 776
    writes = 512 + 1024 + 8
    assert bench.decode_bytes(wl, 0) == reads + writes == 21812
    assert bench.decode_bytes(wl, 15) - bench.decode_bytes(wl, 0) == 15 * 1024
    mean = sum(bench.decode_bytes(wl, c) for c in range(16)) / 16
    assert mean == 29492


def test_flush_and_fp32_bytes_by_hand(bench, wl):
    compact = 512 + 512 + 2048 + 16384
    assert bench.flush_bytes(wl) == (20 + 16 + compact + 16 * 1024) + (compact + 16 + 16) == 55364
    assert bench.fp32_bytes(wl) == 2 * 4 * 128 * 128 + 776 + 512 == 132360
    assert bench.per_step_bytes(wl, "bf16") == 2 * 2 * 128 * 128 + 776 + 512
    assert bench.per_step_bytes(wl, "fp8") == 2 * (128 * 128 + 4 * 128) + 776 + 512


def test_multi_token_bytes_reduce_to_single(bench, wl):
    for c in (0, 7, 15):
        assert bench.multi_decode_bytes(wl, c, 1) == bench.decode_bytes(wl, c)
    # T tokens: the compact state once, T inputs, T outputs and pairs
    d4 = bench.multi_decode_bytes(wl, 4, 4)
    assert d4 == bench.decode_bytes(wl, 4) + 3 * (776 + 512 + 1024)


def test_rates_and_ranks(bench, wl):
    assert bench.whole_job_rate(1000, 1, 1.0) == 1e6
    assert bench.whole_job_rate(1000, 4, 2.0) == 2e6  # every rank's units over the slowest time
    assert bench.max_over_ranks([1.5, 2.0], None, None, 1, "cpu") == [1.5, 2.0]
    assert bench.rank_workload(wl, 0) is wl
    assert bench.rank_workload(wl, 3).seed == wl.seed + 3000


def test_source_hash_ignores_comments(bench):
    a = "int f(int x) { /* doubled\n */ return 2 * x; } // tail\n"
    b = "int f(int x) {\n    return 2 * x;  // twice\n}\n"
    c = "int f(int x) { return 3 * x; }"
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)
    assert len(bench.kernel_source_sha()) == 16


def test_state_memory_figures(bench, wl):
    from linear_attention_recurrent_lq_b200 import build
    build.build()
    from linear_attention_recurrent_lq_b200 import binding as B
    m = bench.state_memory(wl, B)
    assert m["leapquant_blob_bytes"] == 36096
    assert m["leapquant_compact_bytes"] == 20 + 16 + 512 + 512 + 2048 + 16384
    assert m["fp32_blob_bytes"] >= 4 * 128 * 128
    assert 3.0 < m["compact_vs_fp32"] < 3.5
    assert m["layer_leapquant_mb"] == 2048 * 36096 / 1e6


def test_head_token_bytes_and_restore_bytes(bench, wl):
    # window mean of the decode bytes plus the flush spread over the window
    assert bench.head_token_bytes(wl) == (29492 * 16 + 55364) / 16
    # a prefix-cache hit reads and writes the compact part: header 20, meta 16,
    # qs 512, sm 512, compensators 2048, codes 16384
    assert bench.restore_bytes(wl) == 2 * (20 + 16 + 512 + 512 + 2048 + 16384)


def test_cpu_baseline_reports_all_cores_and_one_thread(bench):
    """The oracle leg on a small workload: the contract's keys, a one-thread
    figure beside the all-core one, and the host CPU's model name."""
    import oracle
    from linear_attention_recurrent_lq_b200 import inputs as I
    wl = I.WORKLOADS["gdn_int8_b64h32"].replace(batch=2, heads=4)
    d = I.draw(wl, wl.window)
    r = bench.cpu_baseline(wl, d, 0.2, oracle)
    assert r["kind"] == "oracle" and r["unit"] == "head-tokens/s" and r["value"] > 0
    assert r["cores"] >= 1 and "heads" in r["sample"]
    assert r["one_thread"]["value"] > 0 and r["one_thread"]["unit"] == "head-tokens/s"
    assert r["cpu_model"] is None or isinstance(r["cpu_model"], str)
