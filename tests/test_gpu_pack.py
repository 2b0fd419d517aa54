"""moe_pack_mx_scales: MX FP4 weight scales from row order into the scale-atom
order moe_weights wants, on the device. The result must be the same bytes as
the permutation the harness writes out in Python, and a layer fed the
device-packed scales must give the same bits as one fed the harness's."""
import numpy as np
import pytest
import torch

from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W
from tests import gpu_harness as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,rows,cols", [(1, 128, 128), (3, 256, 384), (2, 2048, 7168)])
def test_pack_matches_the_permutation(n, rows, cols, cuda_device):
    g = torch.Generator(device="cuda").manual_seed(n * 1000 + rows + cols)
    src = torch.randint(0, 255, (n, rows, cols // 32), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
    got = moe.moe_pack_mx_scales(src)
    torch.cuda.synchronize()
    assert torch.equal(got, W.scale_atoms(src))


def test_layer_with_device_packed_scales(cuda_device):
    s = W.spec("decode_fp4", T=32, H=512, E=16, k=4, I=256)
    inp = W.make_inputs(s, seed=9, device="cuda")
    ref = G.run_stages(s, inp, layer=True)
    for m in ("gate", "up", "down"):
        inp[f"s_{m}"] = moe.moe_pack_mx_scales(inp[f"s_{m}_rows"])
    got = G.run_stages(s, inp, layer=True)
    assert G.poll(ref) == 0 and G.poll(got) == 0
    assert torch.equal(ref.out, got.out)
