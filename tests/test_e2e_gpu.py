"""The end-to-end leg of the benchmark stores each step's output in mapped
pinned host memory (the fused kernel writes host memory directly).  Those
bytes must equal the step's output in device memory, for both forms of the
step."""
from __future__ import annotations

import pytest
import torch

import bench
from tests._gpu import raw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["paged", "taps"])
def test_mapped_host_output_equals_device_output(mode):
    dev = torch.device("cuda", 0)
    sets_obj = bench.DecodeSets(2, 6161, dev, max_hist=300, mode=mode)
    m = bench.MappedOut(tuple(sets_obj.sets[0]["out"].shape), torch.bfloat16, dev)
    try:
        import hybrid_sconv_b200 as hs
        s, wl = sets_obj.sets[0], sets_obj.wls[0]
        sets_obj.step(0)              # device output (and the metadata / table)
        torch.cuda.synchronize()
        if mode == "taps":
            hs.sconv_fused_taps(s["x"], sets_obj.weight, sets_obj.cache, s["slot_mapping"],
                                s["taps"], out=m, **wl.kwargs())
        else:
            hs.sconv_fused(s["x"], sets_obj.weight, sets_obj.cache, s["positions"],
                           s["block_table"], s["seq_idx"], s["slot_mapping"], s["query_start"],
                           out=m, **wl.kwargs())
        torch.cuda.synchronize()
        assert torch.equal(m.host_view().view(torch.int16), raw(s["out"]).cpu())
    finally:
        m.free()
