"""The host pipeline (copies of neighbouring steps overlapping the kernels)
gives the same output and KL as the plain forward call, bit for bit, on
every step."""
import pytest
import torch

import bench
import synth
from block_sparse_attention_24_b200.layer import HostPipeline

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


@pytest.mark.parametrize("idx", [0, 1])
def test_host_pipeline_matches_forward(idx):
    w = synth.config(idx)
    V, L, layer, (q, k, v) = bench.build_layer(w, DEV)
    want = layer.forward(q, k, v).clone()
    want_kl = layer.kl_out.clone()
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.zeros(layer.o.shape, dtype=layer.o.dtype).pin_memory()
    hkl = torch.zeros(4, dtype=torch.float32).pin_memory()
    pipe = HostPipeline(layer, q)
    for steps in (1, 3):
        ho.zero_()
        pipe.run((hq, hk, hv), ho, hkl, steps=steps)
        pipe.wait()
        torch.cuda.synchronize()
        V.veda_check_status(L)
        assert torch.equal(ho, want.cpu())
        assert torch.equal(hkl, want_kl.cpu())
