"""Host-side pieces of bench.py that need no GPU: the algorithmic work per stage that the
roofline divides by, and the reading of DRAM traffic from an ncu CSV log."""
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402

STATS = {"n_active_experts": 50, "n_kept": 3000}


def _sum(a, b):
    return {k: a[k] + b[k] for k in a}


def test_layer_work_splits_routed_and_shared_problems():
    """On the tensor-core path the shared experts are a problem of their own: the streaming
    kernels (one launch for both) carry exactly the sum of the two problems' work, and the
    totals count every GEMM once."""
    spec = synth.LayerSpec("w", 1024, 64, 6, 512, n_shared=2, d_ff_shared=256)
    T = 700
    w_tc, tot = bench.layer_work(spec, T, STATS, tc_path=True)
    w_st, _ = bench.layer_work(spec, T, STATS, tc_path=False)
    assert w_st["stream_gateup"] == _sum(w_tc["tc_gateup"], w_tc["tc_shared_gateup"])
    assert w_st["stream_down"]["flops"] == w_tc["tc_down"]["flops"] + w_tc["tc_shared_down"]["flops"]
    # the streaming path keeps expert outputs in fp32, the tensor-core path in fp16
    D, F, Fsh, nk = 1024, 512, 512, STATS["n_kept"]
    assert w_st["stream_down"]["bytes"] - (w_tc["tc_down"]["bytes"] + w_tc["tc_shared_down"]["bytes"]) \
        == 2 * (nk + T) * D
    gemm_flops = sum(w_tc[s]["flops"] for s in ("tc_gateup", "tc_down", "tc_shared_gateup",
                                                 "tc_shared_down", "router_logits"))
    assert gemm_flops == tot["flops"]
    assert w_tc["tc_gateup"]["flops"] == 2 * nk * 2 * F * D
    assert w_tc["tc_shared_gateup"]["flops"] == 2 * T * 2 * Fsh * D


def test_layer_work_joint_launches_carry_both_problems():
    """Small batches run the shared experts inside the routed launches: those stages then carry
    the work of both problems, like the streaming kernels."""
    spec = synth.LayerSpec("w", 1024, 64, 6, 512, n_shared=2, d_ff_shared=256)
    T = 16
    sep, _ = bench.layer_work(spec, T, STATS, tc_path=True)
    jnt, _ = bench.layer_work(spec, T, STATS, tc_path=True, joint=True)
    for s in ("gateup", "down"):
        assert jnt["tc_" + s] == _sum(sep["tc_" + s], sep["tc_shared_" + s])


def test_grad_work_counts_each_array_once():
    """The routing gradient's algorithmic bytes: route_grad reads dy and every Top-K slot's
    expert row and writes dx once; segment routing only changes the routed rows of x that the
    dW pass reads, and the fp32 streaming path keeps expert rows in fp32."""
    spec = synth.SPECS["mixtral"]
    T, D, E, K = 4096, 4096, 8, 2
    w = bench.grad_work(spec, T)
    assert w["route_grad"]["bytes"] == 2 * T * D * 4 + T * K * D * 2 + 2 * E * D * 2 + 36 * T * K
    assert w["route_dw"]["bytes"] == T * D * 2 + 12 * T * K + 8 * D * E
    w32 = bench.grad_work(spec, T, tc_path=False)
    assert w32["route_grad"]["bytes"] - w["route_grad"]["bytes"] == T * K * D * 2
    seg = spec.with_(segment_len=16)
    ws = bench.grad_work(seg, T)
    assert ws["route_grad"]["bytes"] == w["route_grad"]["bytes"]
    assert w["route_dw"]["bytes"] - ws["route_dw"]["bytes"] == (T - T // 16) * D * 2
    assert set(w) == bench.GRAD_STAGES


def test_forward_traffic_hash_ignores_the_gradient_source():
    """Recorded DRAM traffic of a forward kernel stays valid when only the routing gradient's
    source changes; the gradient's own stages hash it."""
    fwd = bench.kernel_source_hash("tc_gateup")
    grad = bench.kernel_source_hash("route_grad")
    assert fwd != grad
    assert bench.kernel_source_hash("tc_down") == fwd
    assert bench.kernel_source_hash("route_dw") == grad


def test_layer_work_without_shared_experts_has_empty_shared_problem():
    spec = synth.LayerSpec("w", 1024, 8, 2, 512)
    w, _ = bench.layer_work(spec, 64, STATS)
    assert w["tc_shared_gateup"] == {"bytes": 0, "flops": 0}
    assert w["tc_shared_down"] == {"bytes": 0, "flops": 0}


def _ncu_csv(path, rows):
    head = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
            '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
            '"Metric Value"')
    lines = ["==PROF== Connected to process 1 (/usr/bin/python3)", head]
    for i, name, metric, unit, value in rows:
        lines.append(f'"{i}","1","python3","127.0.0.1","{name}","1","7","(320, 1, 1)","(148, 1, 1)",'
                     f'"0","10.0","Command line profiler metrics","{metric}","{unit}","{value}"')
    path.write_text("\n".join(lines) + "\n")


def test_record_traffic_reads_ncu_csv(tmp_path, monkeypatch):
    """Per-launch DRAM bytes = read + write of the matching launches, averaged, with ncu's
    unit prefixes and thousands separators; other kernels are ignored; the record only counts
    while the kernel sources are unchanged."""
    # the capture prints template arguments as (int)0; a report read back with ncu -i as 0
    gu = "void beam::tc::tc_grouped_gemm_kernel<(int)0, (int)1, (bool)1>(beam::tc::TcParams)"
    gu2 = "void tc_grouped_gemm_kernel<0, 1, 1>(TcParams)"
    dn = "void beam::tc::tc_grouped_gemm_kernel<(int)2, (int)0, (bool)1>(beam::tc::TcParams)"
    csv = tmp_path / "dram.csv"
    _ncu_csv(csv, [
        (0, gu, "dram__bytes_read.sum", "Gbyte", "1.50"),
        (0, gu, "dram__bytes_write.sum", "Mbyte", "100.00"),
        (1, dn, "dram__bytes_read.sum", "Gbyte", "9.00"),
        (1, dn, "dram__bytes_write.sum", "Gbyte", "9.00"),
        (2, gu2, "dram__bytes_read.sum", "Mbyte", "1,700.00"),
        (2, gu2, "dram__bytes_write.sum", "byte", "0"),
    ])
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda stage="": "abc")
    args = types.SimpleNamespace(record_traffic=str(csv), traffic_kernel=r"tc_grouped_gemm_kernel<(\(int\))?0,",
                                 traffic_stage="tc_gateup", traffic_command="ncu ...",
                                 workload="mixtral-prefill")
    bench.record_traffic(args)
    assert bench.recorded_traffic("tc_gateup", "mixtral-prefill") == 1_650_000_000
    assert bench.recorded_traffic("tc_down", "mixtral-prefill") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda stage="": "changed")
    assert bench.recorded_traffic("tc_gateup", "mixtral-prefill") is None


def test_spread_sample_covers_the_batch():
    s = bench.spread_sample(4096, 2331)
    assert len(s) == 2331 and s[0] == 0 and s[-1] == 4095
    assert (s[1:] > s[:-1]).all()
    assert list(bench.spread_sample(5, 100)) == [0, 1, 2, 3, 4]
    assert list(bench.spread_sample(64, 1)) == [0]


def test_gen_work_counts_generator_matrix_leaders_and_outputs():
    """One cross-layer routing call: the [L*2E][D] matrix and the leaders' rows read once, the
    per-layer routing arrays written once, 2*Tr*D*L*2E FLOPs."""
    spec = synth.SPECS["fine"]                  # D 1536, E 212, K 16, bf16
    w = bench.gen_work(spec, 44, 8192, 16)
    cols = 44 * 2 * 212
    assert w["flops"] == 2 * 512 * 1536 * cols
    assert w["bytes"] == (cols * 1536 * 2 + 512 * 1536 * 2 + 44 * 8192 * 16 * 17 + 44 * 8192 * 8
                          + 44 * 7 * 4)
    one = bench.gen_work(spec, 44, 1, 16)        # one decode token: one leader row
    assert one["flops"] == 2 * 1536 * cols
