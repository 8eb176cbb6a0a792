"""The entry points inside CUDA graphs: the library allocates nothing and
never synchronises, so a fused forward and a backward (including the
backward's zero-fill of grad_value) record into a graph on the capture
stream, and replays give the eager results.  This is the launch-latency path
for small problems such as the decoder (N=2, Lq=300, M=8, D=32, L=4, K=4)."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_backward, msda_backward_fused,
                                                msda_forward_fused)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import F32, GRAD, assert_close, host, to_dev, value_grad_terms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("fused_bwd", [False, True], ids=["split", "fused"])
def test_decoder_step_in_cuda_graph(fused_bwd):
    d = wl.make_inputs(wl.DECODER)
    sh = d["spatial_shapes"]
    value, ref, off, z, g = (to_dev(d[k]) for k in
                             ("value", "reference_points", "offsets", "logits", "grad_out"))
    N, Lq, M, L, K = d["logits"].shape
    out = torch.empty(N, Lq, M * 32, device="cuda")
    loc, attn = torch.empty_like(off), torch.empty_like(z)
    gv = torch.empty(value.shape, device="cuda")
    gl, ga, gr = torch.empty_like(off), torch.empty_like(z), torch.empty_like(ref)

    def step():
        if fused_bwd:
            msda_forward_fused(value, sh, None, ref, off, z, out=out)
            msda_backward_fused(value, sh, None, ref, off, z, g, grad_value=gv,
                                grad_reference_points=gr, grad_offsets=gl, grad_logits=ga)
        else:
            msda_forward_fused(value, sh, None, ref, off, z, out=out,
                               sampling_locations_out=loc, attention_weights_out=attn)
            msda_backward(value, sh, None, loc, attn, g, grad_value=gv,
                          grad_sampling_locations=gl, grad_attention_weights=ga)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = [t.clone() for t in (out, gv, gl, ga)]

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for t in (out, gv, gl, ga):
        t.fill_(float("nan"))  # the replay must rewrite every output
    for _ in range(2):  # a second replay re-zeroes grad_value before accumulating
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager[0]), "graph forward differs from the eager forward"
    assert_close(host(gv), host(eager[1]), rtol=1e-5, atol=1e-6, what="graph grad_value")
    assert torch.equal(gl, eager[2]) and torch.equal(ga, eager[3])
    # and the graph's results are the method's
    ora, _, _ = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                     d["logits"])
    assert_close(host(out), ora, **F32, what="graph out")
    if not fused_bwd:
        oloc = oracle.locations_f32(d["reference_points"], d["offsets"], sh)
        A = oracle.softmax(d["logits"]).astype(np.float32)
        ogv, _, _ = oracle.backward(d["value"], sh, oloc, A, d["grad_out"])
        tv, mv = value_grad_terms(d["value"], sh, oloc, A, d["grad_out"])
        assert_close(host(gv), ogv, **GRAD, what="graph grad_value vs oracle", mass=mv,
                     terms=tv)
    del graph
