"""GPU gate normalisation and Top-K threshold selection against the oracle.

Selection is compared bit for bit (tau, tau_idx and the selected index lists),
both sides working on the same fp32 gate tensor."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, oracle_gates

pytestmark = pytest.mark.gpu


def _gpu_select(logG32, K):
    logG = dev(logG32)
    B, Hkv, T, NB = logG.shape
    tau = torch.empty(B, Hkv, T, device="cuda")
    tidx = torch.empty(B, Hkv, T, dtype=torch.int32, device="cuda")
    sel = torch.empty(B, Hkv, T, max(K - 1, 1), dtype=torch.int32, device="cuda")
    binding.sas_select_threshold(logG, tau, tidx, sel, K)
    torch.cuda.synchronize()
    return tau.cpu().numpy(), tidx.cpu().numpy(), sel.cpu().numpy()


@pytest.mark.parametrize("B,Hkv,T,NB", [(1, 1, 64, 1), (2, 3, 1024, 16), (1, 2, 4096, 64), (1, 1, 2048, 40)])
def test_normalize_matches_oracle(B, Hkv, T, NB):
    s = torch.randn(B, Hkv, T, NB, generator=torch.Generator().manual_seed(T + NB)) * 3
    ref = orc.gate_normalize(s.numpy().astype(np.float64), 64)
    out = torch.empty(B, Hkv, T, NB, device="cuda")
    binding.sas_gate_normalize(dev(s), out)
    got = out.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    if fin.any():
        assert np.max(np.abs(got[fin] - ref[fin])) < 2e-5


@pytest.mark.parametrize("K", [1, 2, 4, 16, 33])
def test_select_bit_exact_random(K):
    w = workloads.custom(B=2, Hkv=2, T=4096, K=K)
    s = torch.randn(w.B, w.Hkv, w.T, w.NB, generator=torch.Generator().manual_seed(K))
    _, logG32, tau, tidx, sel = oracle_gates(s.numpy(), K)
    gt, gi, gs = _gpu_select(logG32, K)
    assert np.array_equal(gt, tau)
    assert np.array_equal(gi, tidx)
    if K > 1:
        assert np.array_equal(gs, sel)


def test_select_adversarial_ties_and_signed_zeros():
    rng = np.random.default_rng(7)
    B, Hkv, T, NB, K = 1, 2, 8192, 128, 16
    vals = rng.integers(-3, 3, size=(B, Hkv, T, NB)).astype(np.float32)   # heavy ties
    zeros = rng.random((B, Hkv, T, NB)) < 0.2
    signs = rng.random((B, Hkv, T, NB)) < 0.5
    vals[zeros & signs] = -0.0
    vals[zeros & ~signs] = 0.0
    c = (np.arange(T) // 64)[None, None, :, None]
    vals = np.where(np.arange(NB)[None, None, None, :] < c, vals, -np.inf).astype(np.float32)
    tau, tidx, sel = orc.select_threshold(vals.astype(np.float64), K, 64)
    gt, gi, gs = _gpu_select(vals, K)
    assert np.array_equal(gt, tau.astype(np.float32))
    assert np.array_equal(gi, tidx)
    assert np.array_equal(gs, sel)


def test_select_full_size_qwen3_4b_layer():
    w = workloads.WORKLOADS["qwen3_4b_t8k"]
    s = workloads.make_training_inputs(w)["s"]
    _, logG32, tau, tidx, sel = oracle_gates(s.numpy(), w.K)
    gt, gi, gs = _gpu_select(logG32, w.K)
    assert np.array_equal(gt, tau) and np.array_equal(gi, tidx) and np.array_equal(gs, sel)
