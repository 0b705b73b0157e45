"""GPU noisy ("full*") selection against the oracle.

The selection is compared bit for bit (logG_sel, tau, tau_idx and the chosen
lists), both sides working on the same fp32 gates and noise; the attention calls
given the noisy selection are held to the forward/backward tolerances."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, oracle_gates
from tests.test_gpu_attention import check_full

pytestmark = pytest.mark.gpu


def gpu_noisy(logG32, noise32, K):
    lg, nz = dev(logG32), dev(noise32)
    B, Hkv, T, NB = lg.shape
    out = torch.full_like(lg, 7.0)
    tau = torch.full((B, Hkv, T), 7.0, device="cuda")
    tidx = torch.full((B, Hkv, T), 7, dtype=torch.int32, device="cuda")
    sel = torch.full((B, Hkv, T, max(K - 1, 1)), 7, dtype=torch.int32, device="cuda")
    binding.sas_select_noisy(lg, nz, out, tau, tidx, sel, K)
    torch.cuda.synchronize()
    return out, tau, tidx, sel


def check_noisy(logG32, noise32, K, same_threshold=True):
    out, tau, tidx, sel = gpu_noisy(logG32, noise32, K)
    r_lg, r_tau, r_tidx, r_sel = orc.select_noisy(logG32, noise32, K, 64)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), r_lg)
    assert np.array_equal(tau.cpu().numpy(), r_tau.astype(np.float32))
    assert np.array_equal(tidx.cpu().numpy(), r_tidx)
    if K > 1:
        assert np.array_equal(sel.cpu().numpy(), r_sel)
    if not same_threshold:
        return out, tau, tidx
    # the threshold of logG_sel is what sas_select_threshold itself finds in it
    t2 = torch.empty_like(tau)
    i2 = torch.empty_like(tidx)
    s2 = torch.empty_like(sel)
    binding.sas_select_threshold(out, t2, i2, s2, K)
    torch.cuda.synchronize()
    assert torch.equal(t2.view(torch.int32), tau.view(torch.int32)) and torch.equal(i2, tidx)
    if K > 1:
        assert torch.equal(s2, sel)
    return out, tau, tidx


@pytest.mark.parametrize("B,Hkv,T,NB,K", [(1, 2, 4096, 64, 16), (2, 1, 2048, 40, 4), (1, 1, 8192, 128, 33),
                                          (1, 2, 1024, 16, 1), (1, 1, 65536, 1024, 64), (1, 1, 512, 8, 16)])
def test_select_noisy_matches_oracle(B, Hkv, T, NB, K):
    rng = np.random.default_rng(T + K)
    s = rng.normal(0.0, 2.0, (B, Hkv, T, NB))
    logG32 = orc.gate_normalize(s, 64).astype(np.float32)
    noise32 = rng.gumbel(0.0, 1.0, (B, Hkv, T, NB)).astype(np.float32)
    check_noisy(logG32, noise32, K)


def test_select_noisy_ties_and_zero_noise():
    rng = np.random.default_rng(5)
    B, Hkv, T, NB, K = 1, 2, 4096, 64, 16
    c = (np.arange(T) // 64)[None, None, :, None]
    m = np.arange(NB)[None, None, None, :]
    lg = rng.integers(-3, 3, size=(B, Hkv, T, NB)).astype(np.float32)
    lg[rng.random(lg.shape) < 0.2] = -0.0
    lg = np.where(m < c, lg, -np.inf).astype(np.float32)
    nz = rng.integers(-1, 2, size=lg.shape).astype(np.float32)
    check_noisy(lg, nz, K)
    # no noise: the plain selection, with logG kept on it
    out, tau, tidx = check_noisy(lg, np.zeros_like(lg), K)
    t0, i0, _ = orc.select_threshold(lg.astype(np.float64), K, 64)
    assert np.array_equal(tau.cpu().numpy(), t0.astype(np.float32)) and np.array_equal(tidx.cpu().numpy(), i0)


@pytest.mark.parametrize("w", [workloads.custom("noisy_g4", "bf16", B=1, Hq=8, Hkv=2, d=128, T=1024, K=4),
                               workloads.custom("noisy_f32", "f32", B=1, Hq=4, Hkv=1, d=64, T=512, K=3)],
                         ids=lambda w: w.name)
def test_full_star_forward_backward(w):
    """The attention calls on the noisy selection: clean gates on the noisy Top-K set."""
    inp = workloads.make_training_inputs(w, seed=2)
    _, logG32, _, _, _ = oracle_gates(inp["s"].numpy(), w.K)
    noise32 = np.random.default_rng(9).normal(0.0, 3.0, logG32.shape).astype(np.float32)
    out, tau, tidx = check_noisy(logG32, noise32, w.K)
    lg_sel = out.cpu().numpy()
    check_full(w, inp, lg_sel, tau.cpu().numpy(), tidx.cpu().numpy())
    # the noisy set differs from the clean one on most rows with a choice to make
    clean = orc.selection_mask(logG32.astype(np.float64), *orc.select_threshold(logG32.astype(np.float64), w.K,
                                                                               w.block)[:2], w.block)
    noisy = orc.selection_mask(lg_sel.astype(np.float64), tau.cpu().numpy(), tidx.cpu().numpy(), w.block)
    assert (clean != noisy).any()


def test_full_star_on_a_packed_sequence():
    """Noisy selection on packed gates: each row chooses inside its own document, and the attention calls
    on the result match the oracle's (on the packed tensors, the chosen set held fixed)."""
    w = workloads.custom("noisy_packed", "bf16", B=1, Hq=8, Hkv=2, d=128, T=2048, K=8)
    cu = [0, 512, 576, 1600, 2048]
    inp = workloads.make_training_inputs(w, seed=6)
    s = dev(inp["s"])
    logG = torch.empty_like(s)
    t0 = torch.empty(1, 2, 2048, device="cuda")
    i0 = torch.empty(1, 2, 2048, dtype=torch.int32, device="cuda")
    binding.sas_gate_normalize_select_varlen(s, logG, t0, i0, None, w.K, cu)
    torch.cuda.synchronize()
    lg32 = logG.cpu().numpy()
    noise32 = np.random.default_rng(11).gumbel(0.0, 1.0, lg32.shape).astype(np.float32)
    out, tau, tidx = check_noisy(lg32, noise32, w.K, same_threshold=False)
    lg_sel = out.cpu().numpy()
    mask = orc.selection_mask(lg_sel.astype(np.float64), tau.cpu().numpy(), tidx.cpu().numpy(), w.block)
    for ts, bs in orc.doc_slices(cu, w.block):
        inside = np.zeros(mask.shape[-1], bool)
        inside[bs] = True
        assert not mask[:, :, ts][..., ~inside].any()
    assert mask.sum(-1).max() <= w.K - 1
    check_full(w, inp, lg_sel, tau.cpu().numpy(), tidx.cpu().numpy())
