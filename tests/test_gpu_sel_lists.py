"""Row lists from the selection's index list (the `sel` argument of sas_fwd / sas_bwd).

The KV-block-outer kernels build, per block, the list of positions that attend
it. Given the selection call's sorted index list they build it from that list
instead of thresholding every row's gates again. The attended set is the same,
so the forward must return exactly the same O and LSE bits, and the backward the
same gradients up to the order of its fp32 reductions. Checked for every
selection call that writes the list: the fused, compact, packed-document and
noisy selections, each also against the oracle on the same inputs."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, max_abs, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _selection(kind, w, s):
    """(gates passed to the attention calls, gate_lse or None, tau, tau_idx, sel, dense logG for the oracle)."""
    if kind == "fused":
        logG, tau, tidx, sel = binding.gate_and_select(s, w.K, want_sel=True)
        return logG, None, tau, tidx, sel, logG
    if kind == "compact":
        lse, tau, tidx, sel = binding.gate_and_select_compact(s, w.K, want_sel=True)
        logG, _, _, _ = binding.gate_and_select(s, w.K)
        return s, lse, tau, tidx, sel, logG
    if kind == "varlen":
        cu = [0, 640, 1024, w.T]
        logG, tau = torch.empty_like(s), torch.empty(w.B, w.Hkv, w.T, device="cuda")
        tidx = torch.empty(w.B, w.Hkv, w.T, dtype=torch.int32, device="cuda")
        sel = torch.empty(w.B, w.Hkv, w.T, w.K - 1, dtype=torch.int32, device="cuda")
        binding.sas_gate_normalize_select_varlen(s, logG, tau, tidx, sel, w.K, cu)
        return logG, None, tau, tidx, sel, logG
    assert kind == "noisy"
    logG = torch.empty_like(s)
    binding.sas_gate_normalize(s, logG)
    noise = torch.from_numpy(np.random.default_rng(5).gumbel(size=tuple(s.shape)).astype(np.float32)).cuda()
    lsel, tau = torch.empty_like(s), torch.empty(w.B, w.Hkv, w.T, device="cuda")
    tidx = torch.empty(w.B, w.Hkv, w.T, dtype=torch.int32, device="cuda")
    sel = torch.empty(w.B, w.Hkv, w.T, w.K - 1, dtype=torch.int32, device="cuda")
    binding.sas_select_noisy(logG, noise, lsel, tau, tidx, sel, w.K)
    return lsel, None, tau, tidx, sel, lsel


@pytest.mark.parametrize("kind", ["fused", "compact", "varlen", "noisy"])
@pytest.mark.parametrize("w", [workloads.custom("sel_g4", "bf16", B=1, Hq=8, Hkv=2, d=128, T=2048, K=6),
                               workloads.custom("sel_g5", "bf16", B=1, Hq=10, Hkv=2, d=128, T=1536, K=17,
                                                s_dist="normal2_planted3")],
                         ids=lambda w: w.name)
def test_lists_from_sel_give_the_same_attention(kind, w):
    inp = workloads.make_training_inputs(w, seed=21)
    Q, K, V, dO, s = (dev(inp[k]) for k in ("Q", "K", "V", "dO", "s"))
    gates, gl, tau, tidx, sel, logG = _selection(kind, w, s)
    outs = []
    for use_sel in (None, sel):
        O, LSE = binding.forward(Q, K, V, gates, tau, tidx, w.K, w.sm_scale, gate_lse=gl, sel=use_sel)
        grads = binding.backward(Q, K, V, O, dO, gates, tau, tidx, LSE, w.K, w.sm_scale, gate_lse=gl, sel=use_sel)
        torch.cuda.synchronize()
        outs.append((O, LSE) + tuple(grads))
    (O0, L0, *g0), (O1, L1, *g1) = outs
    assert torch.equal(O0, O1) and torch.equal(L0, L1), "forward differs with the index list"
    for a, b in zip(g0, g1):
        assert rel_l2(to_np(a), to_np(b)) <= 2e-3
    # and against the oracle, on the GPU's fp32 gates and threshold
    lg = to_np(logG)
    ref = orc.forward_backward(*(to_np(inp[k]) for k in ("Q", "K", "V", "dO")), lg, to_np(tau),
                               tidx.cpu().numpy(), w.block, w.sm_scale)
    assert max_abs(to_np(O1), ref["O"]) <= 2e-2
    for name, got in zip(("dQ", "dK", "dV", "dLogG"), g1):
        assert rel_l2(to_np(got), ref[name]) <= 1e-2, name


def test_sel_entries_outside_their_row_are_reported():
    """An index-list entry that is not an earlier block of its row (here the row's own block, and one past the
    block count) is never used as an index: it is reported as a bounds error in the status word, and the call
    completes (every wait of the call then gives up, so its outputs are not defined). After the word is
    cleared, a call on the same workspace with a correct list is clean and equals the thresholding path."""
    w = workloads.custom("sel_bad", "bf16", B=1, Hq=8, Hkv=2, d=128, T=1024, K=4)
    inp = workloads.make_training_inputs(w, seed=31)
    Q, K, V, s = (dev(inp[k]) for k in ("Q", "K", "V", "s"))
    logG, tau, tidx, sel = binding.gate_and_select(s, w.K, want_sel=True)
    bad = sel.clone()
    bad[0, 0, 200, 0] = 200 // w.block      # the row's own block: not historical
    bad[0, 1, 900, 1] = 1000                # past the block count
    ws = binding.workspace(binding.sas_fwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1))
    O_ref, L_ref = binding.forward(Q, K, V, logG, tau, tidx, w.K, w.sm_scale)
    O = torch.empty_like(Q)
    LSE = torch.empty(w.B, w.Hq, w.T, device="cuda")
    binding.sas_fwd(Q, K, V, logG, tau, tidx, O, LSE, w.K, w.sm_scale, ws, sel=bad)
    torch.cuda.synchronize()
    assert binding.sas_device_status(ws) == 2          # bounds error
    binding.sas_device_status_clear(ws)
    binding.sas_fwd(Q, K, V, logG, tau, tidx, O, LSE, w.K, w.sm_scale, ws, sel=sel)
    torch.cuda.synchronize()
    assert binding.sas_device_status(ws) == 0
    assert torch.equal(O, O_ref) and torch.equal(LSE, L_ref)
