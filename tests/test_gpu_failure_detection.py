"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes gives up, raises the device error word, and the context keeps
working (the wait bound is about two seconds)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_head_b200 import build
    build.build()
    from sparse_attention_indexer_head_b200 import binding
    binding.dsa_device_status(reset=True)
    return binding


def test_bounded_wait_gives_up_and_context_survives(B):
    from sparse_attention_indexer_head_b200 import workloads as W
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    result = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert B.dsa_device_status(reset=True) == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    B.dsa_selftest_bounded_wait(result)
    ev1.record()
    torch.cuda.synchronize()
    assert int(result.item()) == 0                       # the wait reported failure
    assert B.dsa_device_status(reset=True) == 1           # code 1: a bounded wait timed out
    assert 0.2e3 < ev0.elapsed_time(ev1) < 20e3           # it waited, then gave up (ms)
    # the context is usable: a whole step runs clean afterwards
    step = DecodeStep(W.make("tiny"))
    step.run()
    torch.cuda.synchronize()
    assert B.dsa_device_status(reset=True) == 0
    assert (step.outputs_numpy()["token_ids"] >= -1).all()
