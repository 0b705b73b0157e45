"""Failure detection on the GPU without a fault: a bounded wait that runs out.

sas_set_wait_limit_ns shortens every bounded wait of the fwd/bwd tensor-core
kernels. With a limit of 1 ns, a wait that is not satisfied at once gives up:
the CTA records a timeout in the workspace status word, lets the copies and
MMAs it issued finish, frees its tensor memory and returns. The host reads the
status through sas_device_status (SAS_ERR_TIMEOUT); after the limit is restored
and the word cleared, the next call on the same stream and workspace is clean
and matches the oracle."""

import ctypes

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, max_abs, oracle_gates, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _status_call(ws):
    out = ctypes.c_int32(0)
    rc = binding.lib().sas_device_status(binding._ptr(ws), binding._stream(None), ctypes.byref(out))
    return rc, out.value


@pytest.mark.parametrize("which", ["fwd", "bwd"])
def test_wait_limit_expires_then_next_call_is_clean(which):
    w = workloads.custom("tmo", "bf16", B=1, Hq=8, Hkv=2, d=128, T=4096, K=4)
    inp = workloads.make_training_inputs(w, seed=5)
    _, logG32, tau, tidx, _ = oracle_gates(inp["s"].numpy(), w.K)
    Q, K, V, dO = (dev(inp[k]) for k in ("Q", "K", "V", "dO"))
    lg, ta, ti = dev(logG32), dev(tau), dev(tidx)
    O = torch.empty_like(Q)
    LSE = torch.empty(w.B, w.Hq, w.T, device="cuda")
    dQ, dK, dV, dLogG = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(lg)
    ws_f = binding.workspace(binding.sas_fwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1))
    ws_b = binding.workspace(binding.sas_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1))

    def fwd():
        binding.sas_fwd(Q, K, V, lg, ta, ti, O, LSE, w.K, w.sm_scale, ws_f)

    def bwd():
        binding.sas_bwd(Q, K, V, O, dO, lg, ta, ti, LSE, dQ, dK, dV, dLogG, w.K, w.sm_scale, ws_b)

    call, ws = (fwd, ws_f) if which == "fwd" else (bwd, ws_b)
    if which == "bwd":
        fwd()                     # a clean forward first: the backward reads O and LSE
        torch.cuda.synchronize()
        assert binding.sas_device_status(ws_f) == 0
    old = binding.set_wait_limit_ns(1)
    try:
        call()
        torch.cuda.synchronize()
    finally:
        binding.set_wait_limit_ns(old)
    rc, word = _status_call(ws)
    assert word == 1, f"status word {word}: no bounded wait expired"      # SAS_DEV_ERR_TIMEOUT
    assert rc == -4                                                      # SAS_ERR_TIMEOUT
    assert torch.cuda.current_stream().query()                           # the context is usable

    binding.sas_device_status_clear(ws)
    fwd()
    if which == "bwd":
        bwd()
    torch.cuda.synchronize()
    assert binding.sas_device_status(ws_f) == 0 and binding.sas_device_status(ws_b) == 0
    ref = orc.forward_backward(*(to_np(inp[k]) for k in ("Q", "K", "V", "dO")), logG32.astype(np.float64), tau,
                               tidx, w.block, w.sm_scale)
    assert max_abs(to_np(O), ref["O"]) <= 2e-2
    if which == "bwd":
        for name, t in (("dQ", dQ), ("dK", dK), ("dV", dV), ("dLogG", dLogG)):
            assert rel_l2(to_np(t), ref[name]) <= 1e-2, name
