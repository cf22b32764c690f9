"""Failure detection without a GPU fault: a bounded wait that runs out (one block waiting on an
mbarrier phase that nothing completes, through the same wait helper the pipelines use) sets the
timeout bit of the status word; the host reads KDA_ERR_TIMEOUT once (reading clears the word) and
the context stays usable: the next prefill still matches the oracle."""
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
import oracle
from tests._parity import TOL_F32, rel_err

pytestmark = [pytest.mark.gpu, pytest.mark.late]


def test_bounded_wait_gives_up_and_the_context_survives(cuda_device):
    kda.kda_last_device_error()  # start from a clear status word
    kda.kda_selftest_wait_timeout(10_000_000)  # gives up after 10 ms
    assert kda.kda_last_device_error() == kda.KDA_ERR_TIMEOUT
    assert kda.kda_last_device_error() == kda.KDA_OK
    spec = kda_synth.PrefillSpec("t", B=1, T=100, H=2, Dk=32, Dv=32, chunk=32, dtype="f32",
                                 decay="fast", init_std=0.02)
    x = kda_synth.prefill_inputs(spec, 1400, cuda_device)
    o, s = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                             initial_state=x["initial_state"], chunk=32)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    o_ref, s_ref = oracle.recurrent(*(x[n][0].cpu() for n in ("q", "k", "v", "log_alpha",
                                                               "beta")),
                                    initial_state=x["initial_state"].cpu())
    assert rel_err(o[0], o_ref) <= TOL_F32
    assert rel_err(s, s_ref) <= TOL_F32
