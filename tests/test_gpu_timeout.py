"""The tensor-core prefill's failure path: bounded waits that give up.

Every wait of the prefill kernel on one of its pipeline barriers is bounded in
wall time; a CTA whose wait runs out raises PA_DEVERR_TIMEOUT, lets what it
already issued land, frees its tensor memory and exits, so a lost arrival can
never hang the GPU.  Here the bound is set to a nanosecond through the test
hook, so that ordinary waits give up; the call must report PA_ERR_TIMEOUT
through pa_get_error, and the next call on the same device and workspace,
with the default bound back, must match the oracle."""
import pytest
import torch

import paged_kv_gqa_reshape_b200 as pa
import workloads
from tests.gpu_helpers import assert_attention_close, case_to, oracle_varlen, run_varlen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_prefill_wait_timeout_is_reported_and_the_next_call_is_correct():
    cpu = workloads.tiny_prefill()
    dev = case_to(cpu, "cuda")
    ws = pa.varlen_workspace(dev.num_seqs, dev.num_q_tokens, dev.num_q_heads, dev.num_kv_heads,
                             dev.head_dim)
    seen = None
    try:
        pa.set_wait_limit_ns(1)
        for _ in range(3):  # a wait that happens to succeed at once never times out
            run_varlen(dev, workspace=ws)
            st, bits = pa.get_error(ws)
            if st != pa.PA_OK:
                seen = (st, bits)
                break
    finally:
        pa.set_wait_limit_ns(0)
    assert seen is not None, "no wait gave up under a 1 ns bound"
    st, bits = seen
    assert st == pa.PA_ERR_TIMEOUT and bits & pa.DEVERR_TIMEOUT
    assert pa.get_error(ws) == (0, 0)  # the read cleared it
    out, _, _, _ = run_varlen(dev, workspace=ws)
    assert_attention_close(out, oracle_varlen(cpu), what="after a timeout")
    assert pa.get_error(ws) == (0, 0)
