"""GPU forward / backward parity against the oracle.

Both sides get the same inputs: Q/K/V/dO (bf16 values upcast for the oracle)
and the oracle's fp32 gate tensor with its threshold. Tolerances: bf16 outputs
max-abs <= 2e-2 on O, relative L2 <= 1e-2 on dQ/dK/dV/dLogG; the fp32 path is
held to 1e-4."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, max_abs, oracle_gates, rel_l2, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": dict(o=1e-4, rel=1e-4, lse=1e-4), "bf16": dict(o=2e-2, rel=1e-2, lse=1e-2)}


def run_gpu(inp, logG32, tau, tidx, w):
    Q, K, V, dO = (dev(inp[k]) for k in ("Q", "K", "V", "dO"))
    lg, ta, ti = dev(logG32), dev(tau), dev(tidx)
    O, LSE = binding.forward(Q, K, V, lg, ta, ti, w.K, w.sm_scale)
    dQ, dK, dV, dLogG = binding.backward(Q, K, V, O, dO, lg, ta, ti, LSE, w.K, w.sm_scale)
    torch.cuda.synchronize()
    return {k: to_np(v) for k, v in dict(O=O, LSE=LSE, dQ=dQ, dK=dK, dV=dV, dLogG=dLogG).items()}


def check_full(w, inp, logG32, tau, tidx):
    got = run_gpu(inp, logG32, tau, tidx, w)
    ref = orc.forward_backward(*(to_np(inp[k]) for k in ("Q", "K", "V", "dO")), logG32.astype(np.float64), tau,
                               tidx, w.block, w.sm_scale)
    tol = TOL[w.dtype]
    assert max_abs(got["O"], ref["O"]) <= tol["o"], max_abs(got["O"], ref["O"])
    assert max_abs(got["LSE"], ref["LSE"]) <= tol["lse"]
    for k in ("dQ", "dK", "dV", "dLogG"):
        assert rel_l2(got[k], ref[k]) <= tol["rel"], (k, rel_l2(got[k], ref[k]))
    # dLogG is exactly zero off the selection
    mask = orc.selection_mask(logG32.astype(np.float64), tau, tidx, w.block)
    assert np.all(got["dLogG"][~mask] == 0.0)


SMALL = [
    workloads.WORKLOADS["tiny_f32"],
    workloads.custom("bf16_g4", "bf16", B=1, Hq=8, Hkv=2, d=128, T=1024, K=4),
    workloads.custom("bf16_g5_ragged", "bf16", B=1, Hq=10, Hkv=2, d=128, T=512, K=3),
    workloads.custom("bf16_g1", "bf16", B=2, Hq=2, Hkv=2, d=128, T=384, K=2),
    workloads.custom("bf16_g8", "bf16", B=1, Hq=8, Hkv=1, d=128, T=640, K=5, s_dist="normal2_planted3"),
    workloads.custom("f32_d128", "f32", B=1, Hq=4, Hkv=2, d=128, T=320, K=3),
    workloads.custom("bf16_g16", "bf16", B=1, Hq=16, Hkv=1, d=128, T=512, K=4),
    workloads.custom("bf16_g2_k33", "bf16", B=1, Hq=4, Hkv=2, d=128, T=2304, K=33),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fwd_bwd_small(w):
    inp = workloads.make_training_inputs(w, seed=1)
    _, logG32, tau, tidx, _ = oracle_gates(inp["s"].numpy(), w.K)
    check_full(w, inp, logG32, tau, tidx)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_budget_one_current_block_only(dtype):
    w = workloads.custom("k1", dtype, B=1, Hq=4, Hkv=1, d=128, T=512, K=1)
    inp = workloads.make_training_inputs(w, seed=2)
    _, logG32, tau, tidx, _ = oracle_gates(inp["s"].numpy(), w.K)
    check_full(w, inp, logG32, tau, tidx)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unit_gates_full_budget_dense_causal(dtype):
    w = workloads.custom("dense", dtype, B=1, Hq=8, Hkv=2, d=128, T=768, K=12)
    inp = workloads.make_training_inputs(w, seed=3)
    logG32 = np.zeros((w.B, w.Hkv, w.T, w.NB), np.float32)
    tau, tidx, _ = orc.select_threshold(logG32.astype(np.float64), w.K, w.block)
    check_full(w, inp, logG32, tau.astype(np.float32), tidx.astype(np.int32))


def test_single_block_sequence():
    w = workloads.custom("t64", "bf16", B=2, Hq=4, Hkv=1, d=128, T=64, K=4)
    inp = workloads.make_training_inputs(w, seed=4)
    _, logG32, tau, tidx, _ = oracle_gates(inp["s"].numpy(), w.K)
    check_full(w, inp, logG32, tau, tidx)


def _sampled_check(w, inp, logG32, tau, tidx, sel, groups, rows, blocks):
    got = run_gpu(inp, logG32, tau, tidx, w)
    tol = TOL[w.dtype]
    np_in = {k: to_np(inp[k]) for k in ("Q", "K", "V", "dO")}
    G = w.G
    for (b, g) in groups:
        ref = orc.rows_gathered(np_in["Q"], np_in["K"], np_in["V"], np_in["dO"], logG32, sel, b, g, rows, w.block,
                                w.sm_scale)
        hs = slice(g * G, (g + 1) * G)
        assert max_abs(got["O"][b, hs][:, rows], ref["O"]) <= tol["o"]
        assert max_abs(got["LSE"][b, hs][:, rows], ref["LSE"]) <= tol["lse"]
        assert rel_l2(got["dQ"][b, hs][:, rows], ref["dQ"]) <= tol["rel"]
        assert rel_l2(got["dLogG"][b, g][rows], ref["dLogG"]) <= tol["rel"]
        for j in blocks:
            dK, dV = orc.kv_block_gathered(np_in["Q"], np_in["K"], np_in["V"], np_in["dO"], logG32, sel, b, g, j,
                                           w.block, w.sm_scale)
            ks = slice(j * w.block, (j + 1) * w.block)
            assert rel_l2(got["dK"][b, g, ks], dK) <= tol["rel"], ("dK", j)
            assert rel_l2(got["dV"][b, g, ks], dV) <= tol["rel"], ("dV", j)


def test_full_size_qwen3_4b_layer_sampled():
    """The bench workload (B=1, Hq=32, Hkv=8, d=128, T=8192, K=16) at full size;
    the oracle evaluates sampled rows and KV blocks in the gathered form."""
    w = workloads.WORKLOADS["qwen3_4b_t8k"]
    inp = workloads.make_training_inputs(w)
    _, logG32, tau, tidx, sel = oracle_gates(inp["s"].numpy(), w.K)
    rows = np.array([0, 1, 63, 64, 100, 1023, 1024, 4095, 4096, 6000, 8127, 8128, 8191])
    _sampled_check(w, inp, logG32, tau, tidx, sel, [(0, 0), (0, 5)], rows, [0, 1, 64, 126, 127])


def _full_size_sampled(w, groups, rows, blocks, seed=0):
    """Full-size problem on the GPU, checked on sampled (b, g) groups.

    The GPU normalises and selects the gates of every group itself; on the sampled
    groups its gate tensor is compared with the oracle's and then replaced by the
    oracle's fp32 gates, so that both sides attend the same blocks there. The
    oracle evaluates the sampled rows (O, LSE, dQ, dLogG) and KV blocks (dK, dV)
    in the gathered form, one group at a time."""
    inp = workloads.make_training_inputs(w, seed)
    s_cpu = inp["s"]
    G = w.G
    logG, tau, tidx, _ = binding.gate_and_select(dev(s_cpu), w.K)
    ora = {}
    for (b, g) in groups:
        lg64 = orc.gate_normalize(s_cpu[b:b + 1, g:g + 1].numpy().astype(np.float64), w.block)
        got = logG[b, g].cpu().numpy().astype(np.float64)
        fin = np.isfinite(lg64[0, 0])
        assert np.array_equal(np.isneginf(got), np.isneginf(lg64[0, 0]))
        assert np.max(np.abs(got[fin] - lg64[0, 0][fin])) < 2e-5
        lg32 = lg64.astype(np.float32)
        logG[b, g] = dev(lg32[0, 0])
        ta, ti, se = orc.select_threshold(lg32.astype(np.float64), w.K, w.block)
        ora[(b, g)] = (lg32, ta[0, 0].astype(np.float32), ti[0, 0], se)
    sel = torch.empty(w.B, w.Hkv, w.T, w.K - 1, dtype=torch.int32, device="cuda")
    binding.sas_select_threshold(logG, tau, tidx, sel, w.K)
    for (b, g), (_, ta, ti, se) in ora.items():
        assert np.array_equal(tau[b, g].cpu().numpy(), ta)
        assert np.array_equal(tidx[b, g].cpu().numpy(), ti)
        assert np.array_equal(sel[b, g].cpu().numpy(), se[0, 0])
    del sel
    Q, K, V, dO = (dev(inp[k]) for k in ("Q", "K", "V", "dO"))
    O, LSE = binding.forward(Q, K, V, logG, tau, tidx, w.K, w.sm_scale)
    dQ, dK, dV, dLogG = binding.backward(Q, K, V, O, dO, logG, tau, tidx, LSE, w.K, w.sm_scale)
    torch.cuda.synchronize()
    tol = TOL[w.dtype]
    r = torch.as_tensor(rows, device="cuda")
    for (b, g), (lg32, _, _, se) in ora.items():
        hs = slice(g * G, (g + 1) * G)
        grp = [to_np(inp["Q"][b:b + 1, hs]), to_np(inp["K"][b:b + 1, g:g + 1]), to_np(inp["V"][b:b + 1, g:g + 1]),
               to_np(inp["dO"][b:b + 1, hs])]
        ref = orc.rows_gathered(*grp, lg32, se, 0, 0, rows, w.block, w.sm_scale)
        assert max_abs(to_np(O[b, hs][:, r]), ref["O"]) <= tol["o"]
        assert max_abs(to_np(LSE[b, hs][:, r]), ref["LSE"]) <= tol["lse"]
        assert rel_l2(to_np(dQ[b, hs][:, r]), ref["dQ"]) <= tol["rel"]
        assert rel_l2(to_np(dLogG[b, g][r]), ref["dLogG"]) <= tol["rel"]
        for j in blocks:
            rdK, rdV = orc.kv_block_gathered(*grp, lg32, se, 0, 0, j, w.block, w.sm_scale)
            ks = slice(j * w.block, (j + 1) * w.block)
            assert rel_l2(to_np(dK[b, g, ks]), rdK) <= tol["rel"], ("dK", j)
            assert rel_l2(to_np(dV[b, g, ks]), rdV) <= tol["rel"], ("dV", j)


def test_full_size_qwen3_8b_layer_sampled():
    """B=2, Hq=32, Hkv=8, d=128, T=32768, K=32, Student-t selector scores, at full size."""
    w = workloads.WORKLOADS["qwen3_8b_t32k"]
    rows = np.array([0, 1, 63, 64, 2047, 2048, 16384, 20001, 32703, 32704, 32767])
    _full_size_sampled(w, [(0, 0), (1, 7)], rows, [0, 3, 256, 510, 511])


def test_full_size_qwen3_14b_layer_sampled():
    """B=1, Hq=40 (G=5), Hkv=8, d=128, T=65536, K=16, N(0, 1) selector scores, at full size."""
    w = workloads.WORKLOADS["qwen3_14b_t64k"]
    rows = np.array([0, 1, 63, 64, 65, 1000, 4095, 4096, 32768, 50001, 65471, 65472, 65535])
    _full_size_sampled(w, [(0, 3)], rows, [0, 1, 500, 1022, 1023])
