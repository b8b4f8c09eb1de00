"""Failure path on the GPU without a fault: a bounded wait that nothing
satisfies gives up after its limit, the status word reports the timeout, and
the next launches work normally."""
import math

import pytest
import torch

import block_sparse_attention_24_b200 as V
import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    w = synth.config(0)
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device="cuda")
    V.veda_selftest_wait_timeout(L, 50)
    with pytest.raises(V.VedaError) as e:
        V.veda_check_status(L)
    assert e.value.code == V.VEDA_ERR_TIMEOUT
    V.veda_check_status(L)  # cleared
    # the context is still usable: a real launch afterwards succeeds
    q, k, v = (t.cuda() for t in synth.qkv(w, "cpu"))
    qp = torch.empty((1, w.heads, L.n_cap, w.d), dtype=torch.bfloat16, device="cuda")
    V.veda_permute(L, q, qp)
    op = torch.empty_like(qp)
    V.veda_sparse_attn(L, qp, qp, qp, None, None, 0, 1 / math.sqrt(w.d), op)
    V.veda_check_status(L)
    assert torch.isfinite(op.float()).all()


def test_selftest_argument_checks():
    w = synth.config(0)
    L = V.Layer(w.B, w.heads, w.d, w.T, w.H, w.W, w.tile, w.tilings, device="cuda")
    with pytest.raises(V.VedaError) as e:
        V.veda_selftest_wait_timeout(L, 0)
    assert e.value.code == V.VEDA_ERR_INVALID_ARG
