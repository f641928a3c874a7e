"""Host-side helpers of the benchmark (no GPU): percentiles of a timing
sample, the whole-job throughput of N replicas, and the comment-blind source
hash that decides whether the committed DRAM-traffic capture still applies."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def test_percentiles_nearest_rank():
    import bench
    v = [float(x) for x in range(1, 21)]  # 20 samples, unsorted input below
    p = bench.percentiles(list(reversed(v)))
    # nearest rank over 20 samples: index round(q * 19)
    assert p == {"p10": 3.0, "p50": 11.0, "p90": 18.0}
    assert bench.percentiles([2.5]) == {"p10": 2.5, "p50": 2.5, "p90": 2.5}


def test_whole_job_value_is_sum_of_work_over_slowest_rank():
    import bench
    assert abs(bench.whole_job_tflops(3.624e12, 4, 1000.0) - 14.496) < 1e-9


def test_source_hash_ignores_comments_and_whitespace(tmp_path):
    import bench
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f(int x) { return x + 1; }  // add one\n")
    b.write_text("/* header */\nint f(int x) {\n  return x + 1;\n}\n")
    c.write_text("int f(int x) { return x + 2; }\n")
    assert bench._code_sha(str(a)) == bench._code_sha(str(b))
    assert bench._code_sha(str(a)) != bench._code_sha(str(c))


def test_committed_traffic_matches_current_attention_source():
    import bench
    assert bench._ncu_traffic() is not None, "profiles/attn_subset_srsu_2560.traffic.json is stale"


def test_mufu_colimit_at_the_head_dims():
    import bench
    # d = 96: 384 flop per exponential take 384 / 8192 clock of tensor time,
    # an exponential on MUFU 1 / 16: all on MUFU caps the tensor pipe at 75%;
    # with a quarter on the FMA pipe the two times are equal
    c = bench.mufu_colimit(96, 0.75)
    assert c["ceiling_all_on_mufu"] == 0.75 and c["ceiling_as_built"] == 1.0
    assert bench.mufu_colimit(128, 1.0)["ceiling_as_built"] == 1.0
    assert bench.mufu_colimit(64, 1.0)["ceiling_as_built"] == 0.5
