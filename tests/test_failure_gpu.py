"""The bounded-wait failure path of the attention kernel, exercised without any GPU
fault: the library's test switch makes the MMA-issuing thread wait on a barrier that
nothing signals.  That wait gives up after 100 us and records a timeout; the other roles
of every CTA give up their own waits after the 2 s limit, let their TMA copies land and
release tensor memory.  The host must read GQA_ERR_DEVICE_TIMEOUT, and the next normal
call on the same device must match the oracle."""
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, oracle_prefill_args, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def test_attention_wait_timeout_is_reported_and_the_device_stays_usable(gqa):
    inp = synthetic.prefill_inputs(1, 256, 8, 2, seed=300)
    d = to_dev(inp)
    args = (d["q"], d["k"], d["v"], d["pos"], d["qnorm_w"], d["knorm_w"], d["theta"], d["eps"])
    lib = gqa.load()
    assert gqa.device_status() == 0
    lib.gqa_attn_test_stall(1)
    try:
        gqa.prefill(*args)
    finally:
        lib.gqa_attn_test_stall(0)
    torch.cuda.synchronize()
    assert gqa.device_status() == -5   # GQA_ERR_DEVICE_TIMEOUT
    assert gqa.device_status() == 0    # read and cleared
    out = gqa.prefill(*args)
    torch.cuda.synchronize()
    gqa.check_device_status()
    assert_close(out.cpu().numpy(), oracle.prefill(*oracle_prefill_args(inp)), "the call after the timeout")
