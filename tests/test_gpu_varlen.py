"""GPU packed (variable-length) training path against the oracle.

The packed gates and selection come from sas_gate_normalize_select_varlen; the
attention calls and the selector gradient run unchanged on them. Gates within
2e-5 of the oracle; the selection (as the set the threshold keeps) bit-exact
against the oracle's per-document Top-K on the GPU's own fp32 gates; forward and
backward within the tolerances of the other parity tests (bf16: 2e-2 max-abs on
O, 1e-2 relative L2 on the gradients; fp32: 1e-4)."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, max_abs, rel_l2, to_np

pytestmark = pytest.mark.gpu


def gpu_varlen_gates(s, K, cu, want_sel=True):
    B, Hkv, T, NB = s.shape
    logG = torch.full_like(s, 7.0)
    tau = torch.full((B, Hkv, T), 7.0, device="cuda")
    tidx = torch.full((B, Hkv, T), 7, dtype=torch.int32, device="cuda")
    sel = torch.full((B, Hkv, T, max(K - 1, 1)), 7, dtype=torch.int32, device="cuda") if want_sel else None
    binding.sas_gate_normalize_select_varlen(s, logG, tau, tidx, sel, K, cu)
    torch.cuda.synchronize()
    return logG, tau, tidx, sel


def check_gates(s_cpu, K, cu):
    logG, tau, tidx, sel = gpu_varlen_gates(dev(s_cpu), K, cu)
    got = logG.cpu().numpy().astype(np.float64)
    ref = orc.gate_normalize_varlen(s_cpu.numpy().astype(np.float64), cu, 64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), ~fin)
    if fin.any():
        assert np.max(np.abs(got[fin] - ref[fin])) < 2e-5
    mask_gpu = orc.selection_mask(got, tau.cpu().numpy().astype(np.float64), tidx.cpu().numpy(), 64)
    mask_ref = orc.selection_mask_varlen(got, K, cu, 64)
    assert np.array_equal(mask_gpu, mask_ref)
    if K > 1:
        H = K - 1
        want = np.full(sel.shape, -1, dtype=np.int32)
        idx = np.nonzero(mask_ref)
        counts = {}
        for b, g, t, m in zip(*idx):
            k = counts.get((b, g, t), 0)
            want[b, g, t, k] = m
            counts[(b, g, t)] = k + 1
        assert max(counts.values(), default=0) <= H
        assert np.array_equal(sel.cpu().numpy(), want)
    return logG, tau, tidx


@pytest.mark.parametrize("T,NB,K,docs", [
    (4096, 64, 16, [1024, 512, 2560]),
    (2048, 40, 4, [64, 64, 1280, 640]),          # one-block documents, padding columns past T/64
    (8192, 128, 33, [4096, 4096]),
    (1024, 16, 1, [512, 512]),
    (65536, 1024, 16, [8192, 24576, 32768]),     # rows in 32 registers per lane
])
def test_varlen_gates_and_selection(T, NB, K, docs):
    s = torch.randn(2, 2, T, NB, generator=torch.Generator().manual_seed(T + K)) * 2
    check_gates(s, K, np.cumsum([0] + docs).tolist())


def test_varlen_one_document_is_the_plain_fused_call():
    w = workloads.custom("one_doc", "bf16", B=1, Hq=4, Hkv=2, d=128, T=4096, K=16)
    s = dev(torch.randn(1, 2, 4096, 64, generator=torch.Generator().manual_seed(3)))
    got = gpu_varlen_gates(s, w.K, [0, 4096])
    logG = torch.empty_like(s)
    tau = torch.empty(1, 2, 4096, device="cuda")
    tidx = torch.empty(1, 2, 4096, dtype=torch.int32, device="cuda")
    sel = torch.empty(1, 2, 4096, 15, dtype=torch.int32, device="cuda")
    binding.sas_gate_normalize_select(s, logG, tau, tidx, sel, w.K)
    torch.cuda.synchronize()
    for a, b in zip(got, (logG, tau, tidx, sel)):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("w,docs", [
    (workloads.custom("varlen_g4", "bf16", B=1, Hq=8, Hkv=2, d=128, T=2048, K=4), [512, 64, 1024, 448]),
    (workloads.custom("varlen_g8_k8", "bf16", B=2, Hq=8, Hkv=1, d=128, T=1536, K=8), [768, 192, 576]),
    (workloads.custom("varlen_f32", "f32", B=1, Hq=4, Hkv=1, d=64, T=768, K=3), [128, 448, 192]),
], ids=lambda x: getattr(x, "name", "docs"))
def test_varlen_forward_backward_and_gate_grad(w, docs):
    cu = np.cumsum([0] + docs).tolist()
    inp = workloads.make_training_inputs(w, seed=4)
    logG, tau, tidx = check_gates(inp["s"], w.K, cu)
    Q, K, V, dO = (dev(inp[k]) for k in ("Q", "K", "V", "dO"))
    O, LSE = binding.forward(Q, K, V, logG, tau, tidx, w.K, w.sm_scale)
    dQ, dK, dV, dLogG = binding.backward(Q, K, V, O, dO, logG, tau, tidx, LSE, w.K, w.sm_scale)
    ds = binding.gate_grad(logG, dLogG)
    torch.cuda.synchronize()
    lg64 = logG.cpu().numpy().astype(np.float64)
    ref = orc.forward_backward_varlen(*(to_np(inp[k]) for k in ("Q", "K", "V", "dO")), lg64, w.K, cu, w.block,
                                      w.sm_scale)
    tol = {"bf16": (2e-2, 1e-2, 1e-2), "f32": (1e-4, 1e-4, 1e-4)}[w.dtype]
    assert max_abs(to_np(O), ref["O"]) <= tol[0]
    assert max_abs(to_np(LSE), ref["LSE"]) <= tol[1]
    for name, got in (("dQ", dQ), ("dK", dK), ("dV", dV), ("dLogG", dLogG)):
        assert rel_l2(to_np(got), ref[name]) <= tol[2], (name, rel_l2(to_np(got), ref[name]))
    mask = orc.selection_mask_varlen(lg64, w.K, cu, w.block)
    assert np.all(to_np(dLogG)[~mask] == 0.0)
    # selector-score gradient, document by document, against the oracle's Jacobian product
    dl = to_np(dLogG)
    s64 = inp["s"].numpy().astype(np.float64)
    got = to_np(ds)
    for ts, bs in orc.doc_slices(cu, w.block):
        r = orc.gate_grad(s64[:, :, ts, bs], dl[:, :, ts, bs], w.block)
        g = np.exp(orc.gate_normalize(s64[:, :, ts, bs], w.block))
        bound = 3e-5 * (np.abs(dl[:, :, ts, bs]) + g * np.abs(dl[:, :, ts, bs]).sum(-1, keepdims=True))
        assert np.all(np.abs(got[:, :, ts, bs] - r) <= bound + 1e-30)
        other = np.ones(got.shape[-1], bool)
        other[bs] = False
        assert np.all(got[:, :, ts][..., other] == 0.0)


def test_varlen_full_size_qwen3_4b_layer_gates():
    """The bench's packed step (the qwen3_4b_t8k layer as documents of 512, 1536, 1024, 2048 and 3072
    tokens): gates and selection of every row at full size."""
    w = workloads.WORKLOADS["qwen3_4b_t8k"]
    s = workloads.make_training_inputs(w)["s"]
    check_gates(s, w.K, np.cumsum([0, 512, 1536, 1024, 2048, 3072]).tolist())
