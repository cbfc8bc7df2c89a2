"""Failure detection without a GPU fault: a bounded device wait that runs out
reports through the status word and leaves the context usable."""

from __future__ import annotations

import pytest

from lora_adapter_execution_b200 import workloads as wl

from helpers import check_close, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_times_out_and_reports():
    import lora_adapter_execution_b200 as lora
    from lora_adapter_execution_b200 import abi
    assert lora.device_status() == 0
    flag = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    abi.selftest_bounded_wait(20000, flag)          # 20 ms limit, nothing ever arrives
    st = lora.device_status()
    assert st & 0x1, st                              # LORA_DEV_TIMEOUT
    assert int(flag.item()) == 0
    assert lora.device_status() == 0                 # reading clears the word
    # the context is still usable: a forward after the timeout is correct
    import oracle
    inp = wl.make_inputs("tiny")
    plan = lora.Plan(inp.ids, inp.ranks, inp.d_in, inp.d_out)
    Y = torch.empty(inp.T, inp.d_out, dtype=torch.bfloat16, device="cuda")
    lora.linear_fwd(plan, dev_bf16(inp.X), dev_bf16(inp.W), dev_bf16(inp.A_pool), dev_bf16(inp.B_pool),
                    torch.from_numpy(inp.scale).cuda(), Y)
    assert lora.device_status() == 0
    check_close(host_f64(Y), oracle.forward(inp), "after timeout")


def test_selftest_rejects_bad_limit():
    import lora_adapter_execution_b200 as lora
    from lora_adapter_execution_b200 import abi
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(lora.LoraError):
        abi.selftest_bounded_wait(0, flag)
    with pytest.raises(lora.LoraError):
        abi.selftest_bounded_wait(2_000_000, flag)
