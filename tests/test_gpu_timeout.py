"""The bounded-wait exit of the tensor-core prefill, made to run on purpose.

Every wait inside the chunk-scan kernel has a time limit; a wait that gives up
sets a device flag, lets the CTA's copies in flight land, frees its tensor
memory and returns, and ssd_device_status() reports SSD_ERR_TIMEOUT.  The test
switches on ssd_test_stall_prefill, which makes each CTA wait a millisecond on a
barrier that nothing arrives on (a flag nothing sets), so that exit is taken by
every CTA of a launch.  Nothing faults or hangs.  A normal call on the same
device afterwards must still match the oracle, which shows that the aborted
CTAs released what they held."""
import pytest
import torch

import oracle
from gpu_util import assert_close, dev_inputs, gpu_prefill, np64
from selective_state_space_43_b200 import ops
from selective_state_space_43_b200.synth import Dims, make_prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seqlen", [100, 640])   # one partial chunk; five chunks (producers two ahead)
def test_stalled_wait_gives_up_reports_and_recovers(seqlen):
    d = Dims(2, seqlen, 16, 64, 128, 2, 128)
    dims = ops.make_dims(d.batch, d.seqlen, d.nheads, d.headdim, d.d_state, d.ngroups, d.chunk)
    assert ops.prefill_path(dims, torch.bfloat16) == 1
    inp = make_prefill_inputs(d, dtype=torch.bfloat16, seed=301, init_state=True)
    g = dev_inputs(inp)
    ops.device_status()   # start from a clear flag
    L = ops.lib()
    assert L.ssd_test_stall_prefill(1_000_000) == 0   # 1 ms, then give up
    try:
        gpu_prefill(g, d.chunk)
    finally:
        L.ssd_test_stall_prefill(0)
    torch.cuda.synchronize()
    with pytest.raises(ops.SsdError) as err:
        ops.device_status()
    assert err.value.status == 8   # SSD_ERR_TIMEOUT
    ops.device_status()   # the flag was cleared by the read

    y, fs, cs = gpu_prefill(g, d.chunk, y_dtype=torch.float32)
    torch.cuda.synchronize()
    ops.device_status()
    yo, fo, co = oracle.prefill(inp)
    assert_close(np64(y), yo, "y after a stalled call")
    assert_close(np64(fs), fo, "final_state after a stalled call")
