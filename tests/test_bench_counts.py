"""The bench's algorithmic work counters against brute force (CPU).

attended keys per row against the oracle's own selection; the packed-step FLOPs,
the executed (tiled) FLOPs and the HBM byte counts of the gate kernels and the
decode step against explicit loops."""

import math

import numpy as np
import torch

import bench
from gated_block_sparse_flashattention_b200 import workloads
from oracle import sas_oracle as orc


def test_attended_keys_per_row_match_the_oracle_selection():
    w = workloads.custom("cnt", "f32", B=1, Hq=4, Hkv=2, d=64, T=640, K=4)
    s = np.random.default_rng(1).standard_normal((w.B, w.Hkv, w.T, w.NB))
    logG = orc.gate_normalize(s, w.block)
    tau, tidx, _ = orc.select_threshold(logG, w.K, w.block)
    mask = orc.selection_mask(logG, tau, tidx, w.block)
    n = bench.attended_keys_per_row(w.T, w.K, w.block)
    t = np.arange(w.T)
    for g in range(w.Hkv):
        want = (t % w.block) + 1 + w.block * mask[0, g].sum(-1)
        assert np.array_equal(n, want)


def test_packed_step_flops_brute_force():
    w = workloads.custom("cnt", "bf16", B=2, Hq=8, Hkv=2, d=128, T=1024, K=5)
    docs = [128, 64, 512, 320]
    total = 0
    for L in docs:
        for t in range(L):
            total += (t % 64) + 1 + 64 * min(w.K - 1, t // 64)
    fwd, bwd = bench.attended_flops_varlen(w, docs)
    assert fwd == 4.0 * w.d * total * w.B * w.Hq and bwd == 2.5 * fwd
    assert bench.attended_flops_varlen(w, [w.T]) == bench.attended_flops(w)


def test_executed_flops_brute_force():
    w = workloads.custom("cnt", "bf16", B=1, Hq=8, Hkv=2, d=128, T=448, K=4)   # G = 4: q-tiles of 32 positions
    rng = np.random.default_rng(2)
    H = w.K - 1
    sel = np.full((w.B, w.Hkv, w.T, H), -1, dtype=np.int64)
    for g in range(w.Hkv):
        for t in range(w.T):
            c = t // w.block
            if c:
                pick = np.sort(rng.choice(c, size=min(H, c), replace=False))
                sel[0, g, t, :len(pick)] = pick
    fwd, bwd = bench.executed_flops(w, torch.from_numpy(sel))
    mma = 2.0 * 128 * 64 * 128
    P = 32
    f_union = f_kv = b = 0.0
    for g in range(w.Hkv):
        for t0 in range(0, w.T, P):
            rows = range(t0, min(t0 + P, w.T))
            blocks = {t // w.block for t in rows} | {int(m) for t in rows for m in sel[0, g, t] if m >= 0}
            f_union += 2 * mma * len(blocks)
        for j in range(w.NB):
            attend = min(w.block, w.T - j * w.block) + int((sel[0, g] == j).sum())
            f_kv += 2 * mma * math.ceil(attend / P)
            b += 5 * mma * math.ceil(attend / P)
    assert bench.fwd_uses_gather(w)
    assert fwd == f_kv and bwd == b
    # a problem whose per-(b, g) partials exceed the slot budget is counted as the union forward
    big = workloads.custom("cnt", "bf16", B=1, Hq=8, Hkv=2, d=128, T=448, K=4)
    orig = bench.SLOT_BUDGET
    try:
        bench.SLOT_BUDGET = 1
        assert not bench.fwd_uses_gather(big)
        assert bench.executed_flops(big, torch.from_numpy(sel)) == (f_union, b)
    finally:
        bench.SLOT_BUDGET = orig


def test_forward_path_rule_matches_the_library_workspace():
    """bench.fwd_uses_gather follows the library's own choice: the union forward's workspace is the status word
    plus per-q-tile block masks, the gather forward's holds the per-pair partials."""
    from gated_block_sparse_flashattention_b200 import binding
    try:
        binding.lib()
    except RuntimeError:
        import pytest
        pytest.skip("library not built")
    for (B, Hq, Hkv, T, K) in [(1, 32, 8, 8192, 16), (2, 32, 8, 32768, 32), (1, 40, 8, 65536, 16),
                               (1, 4, 1, 262144, 64), (1, 8, 1, 131072, 300), (1, 32, 2, 8192, 100)]:
        w = workloads.custom("rule", "bf16", B=B, Hq=Hq, Hkv=Hkv, d=128, T=T, K=K)
        ws = binding.sas_fwd_workspace_size(B, Hq, Hkv, T, 128, K, binding.SAS_DT_BF16)
        P = (128 // w.G) & ~7
        masks = B * Hkv * ((T + P - 1) // P) * ((w.NB + 31) // 32) * 4
        union_ws = 256 + (masks + 255) // 256 * 256
        assert bench.fwd_uses_gather(w) == (ws != union_ws), (B, Hq, Hkv, T, K)


def test_gate_kernel_byte_counts_brute_force():
    w = workloads.custom("cnt", "f32", B=2, Hq=4, Hkv=3, d=64, T=704, K=4)
    rd_c = sum(min(t // w.block, w.NB) for t in range(w.T)) * 4 * w.B * w.Hkv   # causal part of one fp32 tensor
    full = w.NB * w.T * 4 * w.B * w.Hkv
    thr = w.T * 8 * w.B * w.Hkv                                                   # tau + tau_idx
    assert bench.gate_select_bytes(w) == rd_c + full + thr
    assert bench.gate_select_bytes(w, compact=True) == rd_c + w.T * 4 * w.B * w.Hkv + thr   # row LSE instead of logG
    sel = w.T * (w.K - 1) * 4 * w.B * w.Hkv                                       # the sorted block list
    assert bench.gate_select_bytes(w, compact=True, with_sel=True) == rd_c + w.T * 4 * w.B * w.Hkv + thr + sel
    assert bench.gate_grad_bytes(w) == 2 * rd_c + full
    assert bench.noisy_select_bytes(w) == 2 * rd_c + full + thr


def test_decode_byte_count():
    w = workloads.WORKLOADS["decode_b16_l32k"]
    kv = 2 * w.B * w.Hkv * w.K * w.block * w.d * 2
    assert bench.decode_bytes(w) == kv + 2 * w.B * w.Hq * w.d * 2 + w.B * w.Hkv * w.NB * 4
