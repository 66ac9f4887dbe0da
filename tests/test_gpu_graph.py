"""The forward captured in a CUDA graph: replays give the eager call's
outputs bit for bit, on the three selection paths (cooperative fused
selection, pooled selection with a flag clear, head means with tensor-core
scores), including a replay after the inputs were rewritten in place."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from top_kv_tile_b200 import build
    build.build()
    import top_kv_tile_b200
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return top_kv_tile_b200


@pytest.mark.parametrize("name", ["gqa_small", "cross_small", "long_kv_hs", "ragged"])
def test_forward_graph_replay(nsa, name):
    wl = workloads.get(name)
    inp = workloads.make_inputs(wl)
    dev = torch.device("cuda", 0)
    q, k, v = (inp[x].to(dev) for x in "qkv")
    pins = None if inp["pins"] is None else torch.from_numpy(inp["pins"]).to(dev)
    drops = None if inp["drops"] is None else torch.from_numpy(inp["drops"]).to(dev)
    spec = nsa.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    ws = nsa.workspace(wl.B, wl.Hq, wl.Hkv, wl.Sq, wl.Skv, wl.D, spec, dev)
    keep = torch.empty(wl.B, wl.Hs, wl.NQ, wl.NK, dtype=torch.int8, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(wl.B, wl.Hq, wl.Sq, device=dev)

    def step():
        nsa.nsa_forward(q, k, v, spec, wl.scale, pins, drops, keep_out=keep, out=out, lse=lse, ws=ws)

    # eager reference (also loads the module before capture)
    step()
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    ref = (out.clone(), lse.clone(), keep.clone())

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        out.zero_()
        lse.zero_()
        keep.zero_()
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for _ in range(3):
        out.zero_()
        lse.zero_()
        keep.zero_()
        g.replay()
        torch.cuda.synchronize()
        nsa.nsa_device_status()
        assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(keep, ref[2])

    # new inputs in the same buffers: the replay follows them
    gen = torch.Generator().manual_seed(11)
    q.copy_(torch.randn(q.shape, generator=gen).to(q.dtype))
    step()
    torch.cuda.synchronize()
    ref2 = (out.clone(), lse.clone(), keep.clone())
    assert not torch.equal(ref2[0], ref[0])
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    nsa.nsa_device_status()
    assert torch.equal(out, ref2[0]) and torch.equal(lse, ref2[1]) and torch.equal(keep, ref2[2])
    del g
