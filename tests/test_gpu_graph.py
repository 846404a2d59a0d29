"""The block's forward and backward captured in a CUDA graph.

Every entry point only enqueues work on the caller's stream (kernel launches
with the programmatic-launch attribute, tensor maps encoded on the host), so a
whole fwd+bwd step can be captured once and replayed.  The replay must write
exactly what the eager calls write, bit for bit (same kernels, same inputs),
and must follow new input values written into the captured buffers.
"""

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def test_grg_fwd_bwd_replayed_from_a_cuda_graph(cuda_lib):
    B = cuda_lib
    M, K, d, F, eps = 1024, 512, 768, 1536, 1e-6
    N = 2 * F
    td = {k: v.cuda() for k, v in synth.grg_inputs(M, K, d, F, seed=31).items()}
    lib = B.library()
    ws = B.Workspace(max(lib.coda_grg_fwd_workspace_bytes(M, K, d, N, 0), lib.coda_grg_bwd_workspace_bytes(M, K, d, N)))

    def step(fo=None, bo=None):
        fo = B.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps, out=fo, ws=ws)
        bo = B.grg_bwd(td["dY"], td["X"], td["W1"], fo["H"], fo["r"], fo["AB"], td["g"], td["W2"], out=bo, ws=ws)
        return fo, bo

    fo, bo = step()  # eager: allocates the outputs and sets the kernels up
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in {**fo, **bo}.items()}
    for v in list(fo.values()) + list(bo.values()):
        v.zero_()

    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            step(fo, bo)
    torch.cuda.current_stream().wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    assert ws.query() == (0, 0)
    for k, v in {**fo, **bo}.items():
        assert torch.equal(_bits(v), _bits(ref[k])), k

    # New input values in the captured buffers: the replay follows them.
    td["X"].copy_(synth.grg_inputs(M, K, d, F, seed=32)["X"].cuda())
    g.replay()
    torch.cuda.synchronize()
    got = {k: v.clone() for k, v in {**fo, **bo}.items()}
    fo2, bo2 = step()  # eager on the same new inputs, into fresh outputs
    torch.cuda.synchronize()
    for k, v in {**fo2, **bo2}.items():
        assert torch.equal(_bits(got[k]), _bits(v)), k
    assert not torch.equal(_bits(got["Y"]), _bits(ref["Y"]))


def test_two_streams_run_independent_blocks_concurrently(cuda_lib):
    """Two independent fwd+bwd problems enqueued on two streams at once, each
    with its own workspace: no state is shared between calls, so each result is
    bit-identical to the same problem run alone."""
    B = cuda_lib
    M, K, d, F, eps = 1024, 512, 512, 1024, 1e-6
    N = 2 * F
    lib = B.library()
    nbytes = max(lib.coda_grg_fwd_workspace_bytes(M, K, d, N, 0), lib.coda_grg_bwd_workspace_bytes(M, K, d, N))
    probs = [{k: v.cuda() for k, v in synth.grg_inputs(M, K, d, F, seed=s).items()} for s in (41, 42)]
    wss = [B.Workspace(nbytes), B.Workspace(nbytes)]

    def run(td, ws):
        fo = B.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps, ws=ws)
        bo = B.grg_bwd(td["dY"], td["X"], td["W1"], fo["H"], fo["r"], fo["AB"], td["g"], td["W2"], ws=ws)
        return {**fo, **bo}

    alone = [run(td, ws) for td, ws in zip(probs, wss)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for st in streams:
        st.wait_stream(torch.cuda.current_stream())
    both = []
    for _ in range(3):  # several rounds so the two streams' kernels interleave
        both = []
        for td, ws, st in zip(probs, wss, streams):
            with torch.cuda.stream(st):
                both.append(run(td, ws))
    torch.cuda.synchronize()
    for ws in wss:
        assert ws.query() == (0, 0)
    for a, b in zip(alone, both):
        for k in a:
            assert torch.equal(_bits(a[k]), _bits(b[k])), k
