"""Host logic of the benchmark that needs no GPU: the kernel-source hash that
keys the measured DRAM traffic changes with the code and not with comments,
and the workload description names the step it times."""
import bench
import workloads


def test_code_only_strips_comments_and_keeps_literals():
    src = ('int a = 1; // trailing "comment"\n'
           '/* a block\n   comment */ const char *s = "not // a comment"; char c = \'"\';\n'
           '\n'
           'float b = 2.0f;   \n')
    assert bench._code_only(src) == ('int a = 1;\n const char *s = "not // a comment"; '
                                     'char c = \'"\';\nfloat b = 2.0f;')


def test_code_hash_ignores_comment_edits_only():
    a = "__global__ void k(float *x) { x[0] = 1.0f; } // v1\n"
    b = "// header comment\n__global__ void k(float *x) { x[0] = 1.0f; } /* v2 */\n"
    c = "__global__ void k(float *x) { x[0] = 2.0f; } // v1\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_traffic_key_format_and_sources():
    h = bench.csrc_hash(bench.QUANT_SOURCES)
    assert len(h) == 16 and int(h, 16) >= 0
    assert h == bench.csrc_hash(bench.QUANT_SOURCES)
    assert set(bench.QUANT_SOURCES) <= {"qga_common.cuh", "qga_2bit_tiles.cuh", "qga_2bit.cu"}


def test_workload_config_names_the_step():
    w = workloads.WORKLOADS[bench.WORKLOAD]
    cfg = bench.workload_config(w, 2)
    assert str(w.n) in cfg["workload"].replace(",", "")
    assert "quantize" in cfg["workload"] and "merge" in cfg["workload"]
    assert cfg["parallelism"].startswith("replicas x2")
    assert "L2" in cfg["l2"]


def test_alu_bound_is_the_half_rate_alu_pipe_at_the_max_clock():
    # 148 SMs x 4 sub-partitions x 0.5 warp-instructions per cycle at 1965 MHz
    per_s = 148 * 4 * 0.5 * 1965e6
    r = bench.alu_bound(12.0, 2**27, 200e-6, 148)
    assert abs(r["bound_us"] - 2**27 * 12.0 / 32 / per_s * 1e6) < 1e-9
    assert abs(r["frac"] - r["bound_us"] / 200.0) < 1e-12
    assert bench.alu_bound(None, 2**27, 200e-6, 148) is None


def test_measured_alu_rows_name_every_quantizer_of_the_bench():
    for counts in bench.MEASURED_ALU.values():
        assert all(v > 0 for v in counts.values())
    keys = set().union(*bench.MEASURED_ALU.values())
    assert {"b2", "b4", "b8"} <= keys
    assert {f"b{b1}_{b2}" for b1, b2 in bench.TS_PAIRS} <= keys
