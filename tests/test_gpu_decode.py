"""GPU sparse decode against the oracle (selection bit-exact, output max-abs <= 2e-2)."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, max_abs, to_np

pytestmark = pytest.mark.gpu


def run_decode(inp, w, apply_log_gate=False):
    q, Kc, Vc = dev(inp["q"]), dev(inp["Kc"]), dev(inp["Vc"])
    s, seqlen = dev(inp["s"]), dev(inp["seqlen"])
    o = torch.empty_like(q)
    sel = torch.empty(w.B, w.Hkv, max(w.K - 1, 1), dtype=torch.int32, device="cuda")
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K))
    binding.sas_decode_fwd(q, Kc, Vc, seqlen, s, w.K, o, ws, w.sm_scale, sel_out=sel, apply_log_gate=apply_log_gate)
    torch.cuda.synchronize()
    assert binding.sas_device_status(ws) == 0
    return to_np(o), sel.cpu().numpy()


def check(w, inp, apply_log_gate=False):
    got_o, got_sel = run_decode(inp, w, apply_log_gate)
    ref_o, ref_sel = orc.decode(to_np(inp["q"]), to_np(inp["Kc"]), to_np(inp["Vc"]), inp["seqlen"].numpy(),
                                inp["s"].numpy().astype(np.float64), w.K, w.block, w.sm_scale, apply_log_gate)
    if w.K > 1:
        assert np.array_equal(got_sel, ref_sel)
    tol = 2e-2 if w.dtype == "bf16" else 1e-4
    assert max_abs(got_o, ref_o) <= tol, max_abs(got_o, ref_o)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [1, 3, 16, 40])
def test_decode_small_ragged_lengths(dtype, K):
    w = workloads.custom("dec", dtype, B=5, Hq=8, Hkv=2, d=128, T=2000, K=K, decode=True)
    inp = workloads.make_decode_inputs(w, seed=K, seqlen=[2000, 1, 64, 65, 1333])
    check(w, inp)


def test_decode_log_gate_option():
    w = workloads.custom("dec_lg", "bf16", B=3, Hq=4, Hkv=1, d=128, T=1500, K=5, decode=True)
    inp = workloads.make_decode_inputs(w, seed=9, seqlen=[1500, 700, 90])
    check(w, inp, apply_log_gate=True)


def test_decode_full_size():
    """16 sequences x 1 token over a 32768-token cache, Hq=32, Hkv=8, K=16."""
    w = workloads.WORKLOADS["decode_b16_l32k"]
    inp = workloads.make_decode_inputs(w)
    check(w, inp)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (10, 2), (16, 1)])
def test_decode_group_sizes(dtype, Hq, Hkv):
    """G = 1, 5 and 16 heads per group (the MMA rows past G are padding), ragged lengths incl. 1 and Lmax."""
    w = workloads.custom("dec_g", dtype, B=4, Hq=Hq, Hkv=Hkv, d=128, T=1600, K=6, decode=True)
    inp = workloads.make_decode_inputs(w, seed=Hq, seqlen=[1600, 1, 129, 1000])
    check(w, inp)


@pytest.mark.parametrize("K", [2, 64])
def test_decode_budget_extremes(K):
    """K = 2 (one selected block) and the largest budget, 64, with lengths that leave fewer historical
    blocks than the budget (every historical block taken) and lengths that do not."""
    w = workloads.custom("dec_k", "bf16", B=3, Hq=8, Hkv=2, d=128, T=8192, K=K, decode=True)
    inp = workloads.make_decode_inputs(w, seed=K, seqlen=[8192, 3000, 700])
    check(w, inp)
