"""Host-side pieces of bench.py that need no GPU: the coding label of a workload's streams."""
import torch

import bench
from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth


def test_coding_label():
    w = synth.row_lognormal(128, 1024, seed=3)
    paired = B.stream_info(B.compress(w, 4.0, coding=B.CODING_PAIRED))
    single = B.stream_info(B.compress(w, 4.0, coding=B.CODING_SINGLE))
    assert paired.paired == 1 and single.paired == 0
    assert bench.coding_label([paired, paired]) == "paired"
    assert bench.coding_label([single]) == "single"
    assert bench.coding_label([paired, single]) == "mixed"


def _args(workload, target=None):
    import argparse
    wl = bench.WORKLOADS[workload]
    return argparse.Namespace(workload=workload, target=wl["target"] if target is None else target)


def test_both_arms_state_the_same_config():
    """the GPU arm and the reference arm print one config: the workload and the L2 policy, with
    nothing taken from either arm's own streams"""
    for name in bench.WORKLOADS:
        a = _args(name)
        c1, c2 = bench.bench_config(a, 1), bench.bench_config(a, 1)
        assert c1 == c2 and c1["workload"] == name and c1["parallelism"] == "single"
        assert bench.bench_config(a, 4)["parallelism"] == "replicas"
        keys = {"workload", "shape", "target_bpp", "distribution", "container", "l2", "parallelism"}
        assert set(c1) == (keys | {"tokens"} if bench.WORKLOADS[name].get("scheme") == "linear_fused" else keys)


def test_l2_policy():
    """workloads below twice the L2 rotate over enough copies to exceed it; the others need none"""
    rot, text = bench.l2_policy(_args("lognormal_rows_4096x4096_bf16"))
    nominal = 4096 * 4096 * (4.0 / 8 + 2)
    assert rot == 7 and rot * nominal >= 2 * bench.L2_BYTES and (rot - 1) * nominal < 2 * bench.L2_BYTES
    assert "7 rotating" in text
    for name in ("dit_28blocks_hidden3072_bf16", "outliers_8192x28672_bf16"):
        assert bench.l2_policy(_args(name))[0] == 1
    rot, _ = bench.l2_policy(_args("int8_codes_8192x8192"))
    assert rot * 8192 * 8192 * (3.0 / 8 + 1) >= 2 * bench.L2_BYTES
    # the fused GEMM writes no weight: its copies hold the streams alone (4 bpp of the block's 113 M
    # weights), five of them to exceed twice the L2
    rot, text = bench.l2_policy(_args("linear_fused_dit_block_16tok_bf16"))
    nominal = 3072 * (9216 + 3072 + 12288 + 12288) * 0.5
    assert rot * nominal >= 2 * bench.L2_BYTES and (rot - 1) * nominal < 2 * bench.L2_BYTES
    assert "rotating stream copies" in text
    # the DiT set lists 112 tensors of the four block shapes
    dims = bench.WORKLOADS["dit_28blocks_hidden3072_bf16"]["dims"]
    assert len(dims) == 112 and sum(r * c for r, c in dims) == 28 * 3072 * (9216 + 3072 + 12288 + 12288)


def test_traffic_record_keys():
    """the committed traffic record is looked up by kernel sources and by workload, rate and shape"""
    import argparse
    a = argparse.Namespace(workload="outliers_8192x28672_bf16", target=3.5, shape="8192x8192")
    assert bench.traffic_key(a) == "outliers_8192x28672_bf16@3.5[8192x8192]"
    a = argparse.Namespace(workload="lognormal_rows_4096x4096_bf16", target=4.0, shape=None)
    assert bench.traffic_key(a) == "lognormal_rows_4096x4096_bf16"
    assert len(bench.kernel_source_hash("decode_kernel")) == 16
    # a record taken on other sources is not reported
    assert bench.traffic_for_kernel("no_such_kernel", "lognormal_rows_4096x4096_bf16") is None
