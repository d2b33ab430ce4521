"""The no-hang guarantee of the kernels' copy and tensor-core pipelines: a bounded wait on an
mbarrier phase that nothing completes gives up after its poll limit, reports ISOQ_ST_TIMEOUT
in the status word and lets the kernel finish; a completed phase is seen as completed; the
context stays usable (a quantize + decode right after still matches the oracle)."""
import pytest
import torch

import rotated_bit_kv_isoquant_b200 as iq
import workloads as wl
from _gpu_util import Run, check_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("polls", [1, 4096])
def test_bounded_wait_gives_up_and_reports(oracle, polls):
    status, gave_up, completed = iq.isoq_selftest_bounded_wait(polls=polls)
    assert gave_up and completed
    assert status & iq.ISOQ_ST_TIMEOUT
    cfg = wl.workload(1)
    run = Run(cfg)
    run.prefill()
    Q, out = run.decode()
    torch.cuda.synchronize()
    check_attention(oracle, run, Q, out, cfg.decode_lens())
    assert iq.isoq_get_status(run.cache) == 0


def test_bounded_wait_rejects_bad_arguments():
    lib = iq.raw_lib()
    buf = torch.zeros((2,), dtype=torch.int32, device="cuda")
    assert lib.isoq_selftest_bounded_wait(None, 16, buf.data_ptr(), None) == iq.ISOQ_E_ARG
    assert lib.isoq_selftest_bounded_wait(buf.data_ptr(), 0, buf.data_ptr(), None) == iq.ISOQ_E_ARG
