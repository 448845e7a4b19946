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
