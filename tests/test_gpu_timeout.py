"""Failure detection on the device, without a fault: a bounded wait that runs out.

Every work wait of the grouped GEMM gives up after MOE_WAIT_LIMIT_NS
(default 2 s).  The test-only hook MOE_TEST_STALL=1 makes CTA 0 skip its first
operand load -- a barrier that nothing will complete -- so its MMA warp's wait
runs out at the limit.  The kernel must then raise MOE_FLAG_TIMEOUT, drain the
loads it did issue, free its tensor memory and return; the context stays
usable and the next call on the same stream is correct."""
import numpy as np
import pytest
import torch

import oracle
from tests._util import cuda, gemm_error_bound, normwise, np_, TOL_NORMWISE
from tests.test_gpu_gemm import _gpu_operands, _operands

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("epi", ["f32", "swiglu"])
def test_gemm_wait_runs_out_then_recovers(lib, monkeypatch, epi):
    sizes, N, K = [256, 300, 40], 512, 1024
    a, b, aq, sa, bq, sb, offs, M = _operands(sizes, N, K, seed=17)
    qa, qsa, qb, qsb = _gpu_operands(lib, a, b)
    goffs = cuda(torch.from_numpy(offs))
    single = 0x100

    def run(status):
        if epi == "f32":
            C = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
            lib.fp8_grouped_gemm_blockscaled(len(sizes), goffs, M, N, K, qa, qsa, qb, qsb,
                                             lib.MOE_EPI_F32 | single, C, None, status)
            return C, None
        q = torch.zeros(M, N // 2, dtype=torch.uint8, device="cuda")
        s = torch.zeros(M, N // 256, dtype=torch.float32, device="cuda")
        lib.fp8_grouped_gemm_blockscaled(len(sizes), goffs, M, N, K, qa, qsa, qb, qsb,
                                         lib.MOE_EPI_SWIGLU_REQUANT | single, q, s, status)
        return q, s

    # 1 ms limit and a stage that is never filled: the wait runs out
    monkeypatch.setenv("MOE_WAIT_LIMIT_NS", "1000000")
    monkeypatch.setenv("MOE_TEST_STALL", "1")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    run(st)
    torch.cuda.synchronize()           # returns: no hang, no fault
    assert int(st.item()) & lib.MOE_FLAG_TIMEOUT
    # the next call, with the default limit and no hook, is correct
    monkeypatch.delenv("MOE_TEST_STALL")
    monkeypatch.delenv("MOE_WAIT_LIMIT_NS")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, sc = run(st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    used = int(offs[-1])
    ref = oracle.grouped_gemm_blockscaled(offs, aq, sa, bq, sb)[:used]
    if epi == "f32":
        mag = oracle.grouped_gemm_blockscaled(offs, aq & 0x7F, sa, bq & 0x7F, sb)[:used]
        got = np_(out)[:used]
        assert np.all(np.abs(got - ref) <= gemm_error_bound(mag, K // 128))
    else:
        rq, rs, _ = oracle.swiglu_requant(ref)
        deq_g = oracle.dequant_1x128(np_(out)[:used], np_(sc)[:used])
        assert normwise(deq_g, oracle.dequant_1x128(rq, rs)) < TOL_NORMWISE
