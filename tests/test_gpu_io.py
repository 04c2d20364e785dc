"""GPU check of the overlapped-copy calls (csa2_group_decode_io,
csa2_stack_decode_io): with the step's device inputs zeroed and its
outputs scrambled, the call must copy every layer's inputs in before the
layer reads them and every output out after it is written, so that the
host outputs equal, bit for bit, those of the plain call on device-resident
inputs; eagerly, twice in a row, and replayed from a CUDA graph."""

import pytest
import torch

from fp4_kv_cache_mxfp4_b200 import csa2, workloads
from fp4_kv_cache_mxfp4_b200.device_workload import io_copies, make_device_workload, run_step, run_step_io
from test_gpu_stack import DECODER, ENCODER

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("per_layer", [True, False], ids=["per_layer", "coarse"])
@pytest.mark.parametrize("wl", [workloads.WORKLOADS[0], DECODER, ENCODER], ids=lambda w: w.name)
def test_io_call_matches_the_plain_call(wl, per_layer):
    csa2.load()
    T = make_device_workload(wl, csa2)
    run_step(T, csa2)
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    ref_out = T["outputs"].cpu().clone()
    ref_idx = [L["idx"].cpu().clone() for L in T["layers"] if L["idx"] is not None]

    host_in = T["inputs"].cpu().pin_memory()
    host_out = torch.empty_like(T["outputs"], device="cpu").pin_memory()
    io = csa2.io_args(*io_copies(T, host_in, host_out, per_layer=per_layer))

    def scramble():
        T["inputs"].zero_()
        T["outputs"].fill_(0x7F)
        host_out.fill_(0)
        torch.cuda.synchronize()

    for _ in range(2):
        scramble()
        run_step_io(T, csa2, io)
        torch.cuda.synchronize()
        assert csa2.csa2_device_status() == (0, 0)
        assert torch.equal(host_out, ref_out)
        assert torch.equal(T["inputs"].cpu(), host_in)
        for L, r in zip([L for L in T["layers"] if L["idx"] is not None], ref_idx):
            assert torch.equal(L["idx"].cpu(), r)

    # the same call captured as a graph: the copies are part of it
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run_step_io(T, csa2, io)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_step_io(T, csa2, io)
    torch.cuda.synchronize()
    scramble()
    graph.replay()
    torch.cuda.synchronize()
    assert csa2.csa2_device_status() == (0, 0)
    assert torch.equal(host_out, ref_out)
    del graph
