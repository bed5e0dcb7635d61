"""One process driving the layer on two GPUs in turn.

The library caches per-device state (SM count, function attributes such as
the GEMMs' dynamic shared memory size); a cache keyed on the first device
would make the second device's launches fail.  The same small DeepSeek-shaped
layer (FP8 dispatch, shared expert) runs on cuda:0 and cuda:1 from one thread,
twice each, interleaved, and must give bit-identical outputs on both devices.
"""
import pytest
import torch

import top_routing_expert_warp_b200 as moe
import synth
from gpu_util import LayerRun, upload_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two visible GPUs in one process")
def test_layer_on_two_devices():
    wl = synth.DEEPSEEK.with_(T=600, d=256, H=128, H_shared=128, seed=41)   # 4800 pairs
    runs = []
    for i in (0, 1):
        with torch.cuda.device(i):
            dev, _ = upload_inputs(wl, device=f"cuda:{i}")
            runs.append(LayerRun(wl, dev, device=f"cuda:{i}"))
    outs = {0: [], 1: []}
    for _ in range(2):
        for i in (0, 1):
            with torch.cuda.device(i):
                y = runs[i]()
                assert runs[i].check_status()[0] == moe.MOE_OK
                outs[i].append(y.view(torch.int16).cpu())
    for i in (0, 1):
        assert torch.equal(outs[i][0], outs[i][1])
    assert torch.equal(outs[0][0], outs[1][0])
