"""Compact gates (sas_gate_normalize_select_compact): the per-row log-sum-exp of the
selector scores in place of the dense logG tensor.

The selection must equal the fused call's bit for bit, the rebuilt gates
s - LSE(s) (one fp32 subtraction) must equal its logG bit for bit, and the
forward given (s, LSE) must then return exactly what it returns given logG (the
gradients, reduced with fp32 atomics in a run-dependent order, up to that
rounding). The row LSE itself is compared with the oracle's (fp64)."""

import numpy as np
import pytest
import torch

import bench
from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, max_abs, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K", [1, 4, 16, 33])
def test_compact_selection_and_gates_match_the_fused_call(K):
    w = workloads.custom("cmp", "bf16", B=1, Hq=8, Hkv=2, d=128, T=4096, K=K, s_dist="normal2_planted3")
    s = dev(workloads.make_training_inputs(w, seed=K)["s"])
    logG, tau, tidx, sel = binding.gate_and_select(s, K, want_sel=True)
    lse = torch.empty(w.B, w.Hkv, w.T, device="cuda")
    tau2, tidx2 = torch.empty_like(tau), torch.empty_like(tidx)
    sel2 = torch.empty_like(sel)
    binding.sas_gate_normalize_select_compact(s, lse, tau2, tidx2, sel2, K)
    torch.cuda.synchronize()
    assert torch.equal(tau2, tau) and torch.equal(tidx2, tidx)
    if K > 1:   # with K = 1 nothing is selected and the list has no column to write
        assert torch.equal(sel2, sel)
    c = (torch.arange(w.T, device="cuda") // w.block)[:, None]
    hist = torch.arange(w.NB, device="cuda")[None, :] < c
    rebuilt = s - lse[..., None]                       # fp32, the subtraction the kernels do
    assert torch.equal(rebuilt[..., hist], logG[..., hist])
    ref = orc.gate_lse(s.cpu().numpy(), w.block)
    got = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    assert np.max(np.abs(got[fin] - ref[fin])) < 2e-5


@pytest.mark.parametrize("w", [workloads.WORKLOADS["tiny_f32"],
                               workloads.custom("cmp_bf16", "bf16", B=1, Hq=8, Hkv=2, d=128, T=1024, K=4),
                               workloads.custom("cmp_g5", "bf16", B=1, Hq=10, Hkv=2, d=128, T=512, K=3)],
                         ids=lambda w: w.name)
def test_compact_attention_and_gradients_equal_the_logg_path(w):
    inp = workloads.make_training_inputs(w, seed=9)
    Q, K, V, dO, s = (dev(inp[k]) for k in ("Q", "K", "V", "dO", "s"))
    logG, tau, tidx, _ = binding.gate_and_select(s, w.K)
    lse = torch.empty(w.B, w.Hkv, w.T, device="cuda")
    binding.sas_gate_normalize_select_compact(s, lse, torch.empty_like(tau), torch.empty_like(tidx), None, w.K)
    outs = []
    for gates, gl in ((logG, None), (s, lse)):
        O, LSE = torch.empty_like(Q), torch.empty(w.B, w.Hq, w.T, device="cuda")
        dQ, dK, dV, dLogG, ds = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(s),
                                 torch.empty_like(s))
        wf = binding.workspace(binding.sas_fwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K,
                                                              binding._dtype_code(Q)))
        wb = binding.workspace(binding.sas_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K,
                                                              binding._dtype_code(Q)))
        binding.sas_fwd(Q, K, V, gates, tau, tidx, O, LSE, w.K, w.sm_scale, wf, gate_lse=gl)
        binding.sas_bwd(Q, K, V, O, dO, gates, tau, tidx, LSE, dQ, dK, dV, dLogG, w.K, w.sm_scale, wb, gate_lse=gl)
        binding.sas_gate_grad(gates, dLogG, ds, gate_lse=gl)
        torch.cuda.synchronize()
        assert binding.sas_device_status(wf) == 0 and binding.sas_device_status(wb) == 0
        outs.append((O, LSE, dQ, dK, dV, dLogG, ds))
    # The forward is deterministic: identical bits. The gradients are reduced with fp32 atomics (dQ, and dK/dV
    # in the fp32 kernel), whose order varies from run to run: equal up to that rounding.
    for a, b in zip(outs[0][:2], outs[1][:2]):
        assert torch.equal(a, b)
    for a, b in zip(outs[0][2:], outs[1][2:]):
        assert rel_l2(to_np(a), to_np(b)) <= (2e-3 if w.dtype == "bf16" else 1e-6)
    # and against the oracle, both sides on the same fp32 gate tensor (the one the compact form rebuilds)
    O = to_np(outs[1][0])
    ref = orc.forward_backward(*(to_np(inp[k]) for k in ("Q", "K", "V", "dO")),
                               logG.cpu().numpy().astype(np.float64), tau.cpu().numpy(), tidx.cpu().numpy(),
                               w.block, w.sm_scale)
    tol = 2e-2 if w.dtype == "bf16" else 1e-4
    assert max_abs(O, ref["O"]) <= tol
    for i, k in ((2, "dQ"), (3, "dK"), (4, "dV"), (5, "dLogG")):
        assert rel_l2(to_np(outs[1][i]), ref[k]) <= (1e-2 if w.dtype == "bf16" else 1e-4), k


def test_union_forward_for_a_large_budget_both_gate_forms():
    """32K tokens, 16 query heads per KV head, K = 64: one (b, g) would need more than 8 GiB of per-pair
    partials, so sas_fwd runs the q-tile union forward; checked on sampled rows against the oracle, with
    compact gates giving the same bits."""
    w = workloads.custom("union", "bf16", B=1, Hq=16, Hkv=1, d=128, T=32768, K=64)
    assert not bench.fwd_uses_gather(w)
    inp = workloads.make_training_inputs(w, seed=3)
    Q, K, V, s = (dev(inp[k]) for k in ("Q", "K", "V", "s"))
    logG, tau, tidx, _ = binding.gate_and_select(s, w.K)
    lse = torch.empty(w.B, w.Hkv, w.T, device="cuda")
    binding.sas_gate_normalize_select_compact(s, lse, torch.empty_like(tau), torch.empty_like(tidx), None, w.K)
    O1, L1 = binding.forward(Q, K, V, logG, tau, tidx, w.K, w.sm_scale)
    ws = binding.workspace(binding.sas_fwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1))
    O2, L2 = torch.empty_like(Q), torch.empty_like(L1)
    binding.sas_fwd(Q, K, V, s, tau, tidx, O2, L2, w.K, w.sm_scale, ws, gate_lse=lse)
    torch.cuda.synchronize()
    assert binding.sas_device_status(ws) == 0
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    lg32 = logG.cpu().numpy()
    _, _, sel = orc.select_threshold(lg32.astype(np.float64), w.K, w.block)
    rows = np.array([0, 63, 64, 4000, 4095, 4096, 20000, 32767])
    grp = [to_np(inp["Q"]), to_np(inp["K"]), to_np(inp["V"]), to_np(inp["Q"])]
    ref = orc.rows_gathered(*grp, lg32, sel, 0, 0, rows, w.block, w.sm_scale)
    r = torch.as_tensor(rows, device="cuda")
    assert max_abs(to_np(O1[0][:, r]), ref["O"]) <= 2e-2
    assert max_abs(to_np(L1[0][:, r]), ref["LSE"]) <= 1e-2
