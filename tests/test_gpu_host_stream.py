"""HostStream (batches streamed from pinned host memory, copies overlapping the
neighbouring batches' kernels) returns, for every batch, exactly what one
moe_forward call on the same batch returns: the stream only orders copies."""
import pytest
import torch

from moe_inputs import CONFIGS, generate, shrink

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_54_b200 as moe


@pytest.mark.parametrize("depth", [2, 3])
def test_host_stream_matches_forward(depth):
    shape = shrink(CONFIGS["deepseekmoe"], T=700, d=256, E=16, d_ff=128, d_ff_shared=128)
    dev = torch.device("cuda", 0)
    inp = generate(shape, device=dev)
    cfg = moe.moe_config(shape)
    w = moe.weights_struct(inp.W_r, inp.W1, inp.W2, inp.W3, inp.logit_bias, inp.select_bias,
                           inp.Ws1, inp.Ws3, inp.Ws2)
    n = 5
    g = torch.Generator().manual_seed(7)
    xs = [(torch.randn(shape.T, shape.d, generator=g) * (1 + i)).to(inp.x.dtype).pin_memory()
          for i in range(n)]
    ys = [torch.empty_like(x).pin_memory() for x in xs]
    ls = [torch.empty(2, dtype=torch.float32).pin_memory() for _ in xs]
    hs = moe.HostStream(cfg, dev, w, depth=depth)
    for x, y, l in zip(xs, ys, ls):
        hs.submit(x, y, l)
    hs.drain()
    torch.cuda.synchronize()
    for s in hs.fwd:
        assert moe.moe_device_status(s.ws) == 0
    ref = moe.MoEForward(cfg, dev, keep_routing=False)
    for x, y, l in zip(xs, ys, ls):
        ref(x.to(dev), w)
        torch.cuda.synchronize()
        assert torch.equal(y, ref.y.cpu())
        assert l[0].item() == ref.aux.item() and l[1].item() == ref.zloss.item()
