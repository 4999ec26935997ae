"""Host-side pieces of bench.py that need no GPU: the launch count it reports
matches the per-step launch lists taken with ncu (bf16_e8: 18 launches; the
MXFP8 E=128 workload with the unfused dispatch: 27)."""

import bench
from mixture_experts_layer_offsets_b200 import inputs


def test_launch_counts_match_the_measured_launch_lists():
    c = inputs.CONFIGS
    assert bench.launches_per_step(c["bf16_e8"], None, False, False) == 18
    assert bench.launches_per_step(c["mxfp8_e128"], None, False, False) == 27
    # the fused dispatch trades one permute and three forward launches for four
    assert bench.launches_per_step(c["mxfp8_e128"], None, False, True) == 27 - 1 - 3 + 4 - 0
    assert bench.launches_per_step(c["bf16_e8"], None, True, False) == 19
