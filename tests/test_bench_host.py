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
