"""GPU selector-score gradient and the fused normalise+select against the oracle.

The fused call must reproduce the two separate calls bit for bit (same
arithmetic, same summation order). The gradient
ds_m = dLogG_m - g_m * sum_{l<c} dLogG_l (SAS paper, Appendix D.3) is checked
element by element against the oracle's Jacobian product with an fp32 bound:
the row sum of up to NB terms and the exp of an fp32 log gate each carry a few
units in the last place, so |err_m| <= 3e-5 * (|dLogG_m| + g_m * sum_l |dLogG_l|).
"""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, oracle_gates

pytestmark = pytest.mark.gpu


def _outputs(s, K, want_sel):
    """Output buffers filled with a poison value, so both forms must write the same entries."""
    B, Hkv, T, NB = s.shape
    logG = torch.full_like(s, 7.0)
    tau = torch.full((B, Hkv, T), 7.0, device="cuda")
    tidx = torch.full((B, Hkv, T), 7, dtype=torch.int32, device="cuda")
    sel = torch.full((B, Hkv, T, max(K - 1, 1)), 7, dtype=torch.int32, device="cuda") if want_sel else None
    return logG, tau, tidx, sel


def _separate(s, K, want_sel):
    logG, tau, tidx, sel = _outputs(s, K, want_sel)
    binding.sas_gate_normalize(s, logG)
    binding.sas_select_threshold(logG, tau, tidx, sel, K)
    return logG, tau, tidx, sel


def _fused(s, K, want_sel):
    logG, tau, tidx, sel = _outputs(s, K, want_sel)
    binding.sas_gate_normalize_select(s, logG, tau, tidx, sel, K)
    return logG, tau, tidx, sel


def _bits(t):
    return t.cpu().contiguous().view(torch.int32).numpy()


@pytest.mark.parametrize("B,Hkv,T,NB,K,want_sel", [
    (1, 1, 64, 1, 4, True),          # no historical block anywhere
    (2, 3, 1024, 16, 4, True),
    (1, 2, 4096, 64, 16, True),
    (1, 1, 2048, 40, 33, True),      # NB not a multiple of 32, padding blocks past T/64
    (1, 2, 8192, 128, 16, False),    # the training layer's row length, no index list
    (1, 2, 8192, 128, 1, True),      # K = 1: current block only
    (1, 1, 65536, 1024, 64, True),   # the longest row the registers hold
    (1, 1, 69632, 1088, 16, True),   # longer rows: the two-kernel form
])
def test_fused_normalize_select_equals_separate_calls(B, Hkv, T, NB, K, want_sel):
    g = torch.Generator().manual_seed(T + NB + K)
    s = dev(torch.randn(B, Hkv, T, NB, generator=g) * 2)
    ref = _separate(s, K, want_sel)
    got = _fused(s, K, want_sel)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(got[0]), _bits(ref[0]))
    assert np.array_equal(_bits(got[1]), _bits(ref[1]))
    assert torch.equal(got[2], ref[2])
    if want_sel:
        assert torch.equal(got[3], ref[3])


def test_fused_normalize_select_matches_oracle_full_size():
    w = workloads.WORKLOADS["qwen3_4b_t8k"]
    s = workloads.make_training_inputs(w)["s"]
    logG64, _, _, _, _ = oracle_gates(s.numpy(), w.K)
    logG, tau, tidx, sel = binding.gate_and_select(dev(s), w.K, want_sel=True)
    got = logG.cpu().numpy().astype(np.float64)
    fin = np.isfinite(logG64)
    assert np.array_equal(np.isneginf(got), ~fin)
    assert np.max(np.abs(got[fin] - logG64[fin])) < 2e-5
    # the selection is the oracle's own on the GPU's fp32 gates
    o_tau, o_tidx, o_sel = orc.select_threshold(got, w.K, w.block)
    assert np.array_equal(tau.cpu().numpy(), o_tau.astype(np.float32))
    assert np.array_equal(tidx.cpu().numpy(), o_tidx)
    assert np.array_equal(sel.cpu().numpy(), o_sel)


def _check_gate_grad(s, dl, block=64):
    """GPU ds on the oracle's fp32 gates against the oracle's ds, element by element."""
    logG64 = orc.gate_normalize(s, block)
    ds = torch.full(s.shape, 7.0, device="cuda")
    binding.sas_gate_grad(dev(logG64.astype(np.float32)), dev(dl.astype(np.float32)), ds)
    got = ds.cpu().numpy().astype(np.float64)
    ref = orc.gate_grad(s, dl.astype(np.float32).astype(np.float64), block)
    fin = np.isfinite(logG64)
    g = np.exp(logG64)
    row_abs = np.abs(np.where(fin, dl, 0.0)).sum(-1, keepdims=True)
    bound = 3e-5 * (np.abs(dl) + g * row_abs)
    assert np.all(got[~fin] == 0.0)
    assert np.all(np.abs(got - ref) <= bound + 1e-30)
    return got, fin


@pytest.mark.parametrize("B,Hkv,T,NB", [(1, 1, 64, 1), (2, 3, 1024, 16), (1, 2, 4096, 64), (1, 1, 2048, 40),
                                        (1, 1, 4096, 100)])
def test_gate_grad_matches_oracle(B, Hkv, T, NB):
    rng = np.random.default_rng(T * 7 + NB)
    s = rng.normal(0.0, 2.0, (B, Hkv, T, NB))
    dl = rng.normal(0.0, 1.0, (B, Hkv, T, NB))    # non-zero past c_t too: ignored by both sides
    got, fin = _check_gate_grad(s, dl)
    # single-block rows (c_t = 1): g = 1 exactly, so ds = dLogG - dLogG = 0
    t = np.arange(T)
    one = (t // 64 == 1) & (NB >= 1)
    assert np.all(got[:, :, one, :] == 0.0)


def test_gate_grad_full_size_qwen3_4b_layer():
    w = workloads.WORKLOADS["qwen3_4b_t8k"]
    s = workloads.make_training_inputs(w)["s"].numpy().astype(np.float64)
    rng = np.random.default_rng(3)
    # sparse dLogG as the backward leaves it: non-zero on K-1 blocks per row
    dl = np.zeros(s.shape)
    sel = rng.random(s.shape) < (w.K - 1) / w.NB
    dl[sel] = rng.normal(0.0, 1e-3, int(sel.sum()))
    got, fin = _check_gate_grad(s, dl)
    # rows sum to zero within the bound's scale
    rs = np.abs(np.where(fin, got, 0.0).sum(-1))
    assert np.all(rs <= 1e-4 * np.abs(np.where(fin, dl, 0.0)).sum(-1) + 1e-12)
