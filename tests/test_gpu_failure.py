"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait inside the library's kernels gives up after a limit, records
NSA_ERR_TIMEOUT and the wait's site code in the device error word and
returns. nsa_selftest_timeout launches a kernel whose one wait (through the
same helpers) is on a condition nothing satisfies, with a short limit; the
host then reads the timeout through nsa_device_status, and the next call of
the whole path runs normally and still matches the oracle.
"""
import pytest
import torch

import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from top_kv_tile_b200 import build
    build.build()
    import top_kv_tile_b200
    assert torch.cuda.is_available()
    return top_kv_tile_b200


def _forward_matches_oracle(nsa):
    wl = workloads.get("cross_small")
    inp = workloads.make_inputs(wl)
    q, k, v = (inp[x].cuda() for x in "qkv")
    pins = torch.from_numpy(inp["pins"]).cuda()
    drops = torch.from_numpy(inp["drops"]).cuda()
    spec = nsa.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    keep = torch.empty(wl.B, wl.Hs, wl.NQ, wl.NK, dtype=torch.int8, device="cuda")
    out, lse = nsa.nsa_forward(q, k, v, spec, wl.scale, pins, drops, keep_out=keep)
    nsa.nsa_device_status()  # raises if any wait of the path gave up
    qn, kn, vn = (inp[x].double().numpy() for x in "qkv")
    ospec = oracle.SparseSpec(wl.budget, wl.block_q, wl.block_kv, wl.head_shared, wl.force)
    okeep, scores, plan = oracle.select_blocks(qn, kn, ospec, inp["pins"], inp["drops"], return_scores=True)
    gk = keep.cpu().numpy()
    parity.check_keep_rows(gk, okeep, scores, plan)
    ro, rl = oracle.block_sparse_attention(qn, kn, vn, okeep, wl.block_q, wl.block_kv, wl.scale)
    parity.check_attention(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl)


@pytest.mark.parametrize("which,site", [(0, 0x70), (1, 0x71)])
def test_bounded_wait_runs_out_and_the_context_stays_usable(nsa, which, site):
    nsa.nsa_device_status()  # start from a clear error word
    nsa.nsa_selftest_timeout(which, 20000)  # about 10 us of SM clock
    with pytest.raises(nsa.NsaError) as e:
        nsa.nsa_device_status()
    assert e.value.status == nsa.NSA_ERR_TIMEOUT
    assert f"wait site {site}" in str(e.value)
    # the status call cleared the word: nothing is left over
    nsa.nsa_device_status()
    # the context is usable and the path still matches the oracle
    _forward_matches_oracle(nsa)
