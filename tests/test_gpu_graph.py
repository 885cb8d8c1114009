"""The C ABI calls are stream-ordered and synchronise nothing on the host, so a
whole step (solattn_pool + solattn_forward, and solattn_dense) can be captured
into a CUDA graph and replayed: the replay gives, bit for bit, the results of
the eager calls, and a second replay on new inputs copied into the captured
buffers follows them."""
import pytest
import torch

import block_sparse_attention_cov_b200 as sa
from block_sparse_attention_cov_b200.build import build
from block_sparse_attention_cov_b200.inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build()


def test_step_captured_in_a_cuda_graph_replays_bitwise():
    wl = Workload("g", 1, 4, 128, (1, 1, 64 * 40 + 9))
    q, k, v = (x.cuda() for x in make_qkv(wl, seed=31))
    beta = 0.6
    # eager reference (also warms the library up: first-call lookups happen here)
    st_e = sa.pool(q, k, v)
    ref = sa.forward(q, k, v, st_e, beta)
    ref_dense = sa.dense(q, k, v)
    torch.cuda.synchronize()

    st = sa.pool(q, k, v)
    ws = sa.workspace()
    out, lse = torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    dens = torch.empty_like(ref[2])
    dout, dlse = torch.empty_like(q), torch.empty_like(lse)
    ws_d = sa.workspace()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            sa.pool(q, k, v, st)
            sa.forward(q, k, v, st, beta, out=out, lse=lse, density=dens, ws=ws)
            sa.dense(q, k, v, out=dout, lse=dlse, ws=ws_d)
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    assert sa.status(ws) == 0 and sa.status(ws_d) == 0
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(dens, ref[2])
    assert torch.equal(dout, ref_dense[0]) and torch.equal(dlse, ref_dense[1])

    # new inputs in the captured buffers: the replay follows them
    q2, k2, v2 = (x.cuda() for x in make_qkv(wl, seed=32))
    st2 = sa.pool(q2, k2, v2)
    ref2 = sa.forward(q2, k2, v2, st2, beta)
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    graph.replay()
    torch.cuda.synchronize()
    assert sa.status(ws) == 0
    assert torch.equal(out, ref2[0]) and torch.equal(lse, ref2[1]) and torch.equal(dens, ref2[2])
