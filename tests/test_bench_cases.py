"""Host logic of the bench's workload choice (no GPU): the measured case is the
128K prefill with the 64-sequence decode; "small" is the ncu-capture instance of
the same kernels; "long" is the 2^20-token chunked prefill and decode pair."""
import bench
from synth import WORKLOADS


def test_full_case_is_the_measured_workload():
    wp, wd = bench.cases("full")
    assert (wp.name, wd.name) == ("prefill_128k", "decode_b64_64k_128k")
    assert wp.n_q == wp.n_kv == 131072 and wd.batch == 64


def test_small_case_keeps_the_shapes_of_the_measured_one():
    wp, wd = bench.cases("small")
    full_p, full_d = bench.cases("full")
    assert wp.name == "prefill_32k" and wd.batch == 8 and wd.name == "decode_b8"
    for f in ("h_q", "h_kv", "d", "d_idx", "block_k", "topk"):
        assert getattr(wp, f) == getattr(full_p, f) and getattr(wd, f) == getattr(full_d, f)


def test_long_case_is_a_chunk_at_the_end_of_a_million_tokens():
    wp, wd = bench.cases("long")
    assert wp is WORKLOADS["chunked_prefill_1m"] and wd is WORKLOADS["decode_b8_1m"]
    assert wp.n_kv == 1 << 20 and wp.n_q == 8192 and wd.batch == 8


def test_ranks_get_independent_seeds_of_the_same_shape():
    a_p, a_d = bench.rank_workloads("long", 0)
    b_p, b_d = bench.rank_workloads("long", 3)
    assert (a_p.n_q, a_p.n_kv, a_d.batch) == (b_p.n_q, b_p.n_kv, b_d.batch)
    assert b_p.seed - a_p.seed == 3000 and b_d.seed - a_d.seed == 3000


def test_profiling_cases_exceed_the_l2_with_few_gb():
    wp, wd = bench.cases("prof")
    assert wp.n_q == 4096 and wp.n_kv == 65536 and wd.batch == 8
    wp2, wd2 = bench.cases("prof_decode")
    assert wp2 == wp and wd2.batch == 64 and (wd2.kv_min, wd2.kv_max) == (16384, 32768)
    # index keys: 128 B per token, above the 126 MB L2 even at the shortest lengths
    assert wd2.batch * wd2.kv_min * wd2.d_idx * 2 > 126 * 2 ** 20
