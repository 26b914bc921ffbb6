"""Failure detection on the GPU without a fault: a bounded mbarrier wait that
nothing completes gives up, the kernel ends, the host reads AVQ_ERR_TIMEOUT
from the device error word, and the context keeps working."""
import pytest

import adaptive_vector_quantized_b200 as avq
from adaptive_vector_quantized_b200 import synth

from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    avq.avq_check_device()  # clean to start with
    avq.avq_selftest_wait(2000)
    with pytest.raises(avq.AVQError) as ei:
        avq.avq_check_device()
    assert ei.value.status == avq.AVQ_ERR_TIMEOUT
    avq.avq_check_device()  # the word was cleared
    # the context is still usable: a small forward still matches the oracle
    inp = synth.make_inputs(synth.get_config("vit", B=1, H=2), 1001)
    res = gh.gpu_forward(inp)
    gh.check_forward(inp, res)
    avq.avq_check_device()
