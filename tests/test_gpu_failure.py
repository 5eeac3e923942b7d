"""Failure detection on the GPU without a GPU fault: the library's bounded
mbarrier wait is made to run out (an mbarrier that nothing arrives at) and
must report TB_DEV_ERR_TIMEOUT through the status word, after which the
context keeps working.  The positive control arrives and reports nothing."""
import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import assert_close_rows, config_of, make_layer

pytestmark = pytest.mark.gpu

TIMEOUT = 0x4  # TB_DEV_ERR_TIMEOUT
WL = S.TINY_F32


def test_bounded_wait_completes_when_the_arrival_comes():
    ctx = TB.Context(config_of(WL))
    ctx.selftest_bounded_wait(20_000_000, arrive=True)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0


def test_bounded_wait_times_out_reports_and_leaves_the_context_usable():
    ctx = TB.Context(config_of(WL))
    ctx.selftest_bounded_wait(20_000_000, arrive=False)   # about 10 ms of SM cycles
    torch.cuda.synchronize()
    assert ctx.check_status() & TIMEOUT
    assert ctx.check_status() == 0                        # reading clears the word
    # the same context still computes correctly: dense attention of a layer
    ld = make_layer(ctx, WL, 0, list(WL.seq_lens))
    out = torch.empty((WL.B, WL.Hq, WL.D), device="cuda")
    ctx.sparse_attn(0, ld.q_dev, None, TB.TB_MASK_DENSE, out)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    L = WL.seq_lens[0]
    for h in range(WL.Hq):
        ref, _ = O.attend(ld.q[0, h], ld.K[0, h // 2, :L], ld.V[0, h // 2, :L], np.arange(L), 1 / np.sqrt(WL.D))
        assert_close_rows(out.cpu().numpy()[0, h][None], ref[None], "f32", f"h{h}")


def test_bounded_wait_rejects_out_of_range_limits():
    ctx = TB.Context(config_of(WL))
    with pytest.raises(TB.TBError):
        ctx.selftest_bounded_wait(0, arrive=False)
    with pytest.raises(TB.TBError):
        ctx.selftest_bounded_wait(10**12, arrive=False)
