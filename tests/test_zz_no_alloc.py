"""w4a_gemv_noalloc: the GEMV with the library's fixed scratch instead of a
caller workspace.  It runs the same kernel and split as w4a_gemv, so its
results must equal w4a_gemv's bit for bit, on two calls in a row (the scratch
keeps the previous call's contents; each call clears its control words).
Collected last, so it also runs after every other GPU test in the session."""
import pytest
import torch

from w4_weight_only_b200 import synth

pytestmark = pytest.mark.gpu


def _api():
    from w4_weight_only_b200 import api, _abi
    return api, _abi


@pytest.mark.parametrize("n,k,batch,epi", [(768, 512, 1, 0), (3072, 512, 5, 2), (5120, 27648, 1, 0),
                                           (55296, 5120, 1, 2), (1024, 1536, 3, 1), (7168, 5120, 4, 0)])
def test_noalloc_equals_workspace_gemv_twice(built_lib, cuda, n, k, batch, epi):
    api, abi = _api()
    W, x = synth.gemv_case(30, n, k, batch, "cuda")
    lin = api.quantize_linear(W, row_interleave=(epi == abi.EPI_SILU_MUL))
    ref = api.gemv(lin, x, epilogue=epi)
    for _ in range(2):
        got = api.gemv_noalloc(lin, x, epilogue=epi)
        api.check_noalloc()  # the scratch's error word: no wait ran out
        if epi == abi.EPI_SUMSQ:
            assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
        else:
            assert torch.equal(got, ref)


def test_noalloc_rejects_oversized_scratch(built_lib, cuda):
    """gate/up at batch 16 needs more than the fixed scratch: refused, and the
    next call that fits still works."""
    api, abi = _api()
    W, x = synth.gemv_case(31, 55296, 5120, 16, "cuda")
    lin = api.quantize_linear(W)
    need = api.gemv_workspace(lin, 16).numel()
    assert need > abi.NOALLOC_SCRATCH_BYTES
    with pytest.raises(abi.W4AError) as e:
        api.gemv_noalloc(lin, x)
    assert e.value.code == abi.ERR_WORKSPACE
    ref = api.gemv(lin, x[:1])
    assert torch.equal(api.gemv_noalloc(lin, x[:1]), ref)
    api.check_noalloc()


def test_noalloc_error_word_is_readable(built_lib, cuda, monkeypatch):
    """A wait that runs out inside w4a_gemv_noalloc lands in the fixed
    scratch's error word, which w4a_check(NULL, 0, stream) reads; the next
    call clears it and succeeds.  (The waits of a CTA for the others are
    bounded to a few dozen cycles here, so the grid barrier between the GEMV
    and its reduction cannot complete in time.)"""
    api, abi = _api()
    W, x = synth.gemv_case(32, 1024, 1536, 3, "cuda")
    lin = api.quantize_linear(W)
    ref = api.gemv(lin, x, epilogue=abi.EPI_SUMSQ)
    monkeypatch.setenv("W4A_BARRIER_WAIT_CYCLES", "32")
    api.gemv_noalloc(lin, x, epilogue=abi.EPI_SUMSQ)
    with pytest.raises(abi.W4AError) as e:
        api.check_noalloc()
    assert e.value.code == abi.ERR_TIMEOUT
    monkeypatch.delenv("W4A_BARRIER_WAIT_CYCLES")
    got = api.gemv_noalloc(lin, x, epilogue=abi.EPI_SUMSQ)
    api.check_noalloc()
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
