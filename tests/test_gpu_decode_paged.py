"""GPU decode over a paged KV cache, and the long-row selection, against the oracle.

Selection is compared bit for bit; outputs within 2e-2 max-abs (bf16 storage).
The paged call must also equal the contiguous call on the same logical cache bit
for bit: both run the same kernels, only the addresses of the copies differ."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import max_abs, to_np

pytestmark = pytest.mark.gpu

SAS_DEV_ERR_BOUNDS = 2


def _to_dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def run_paged(d, w, apply_log_gate=False):
    o = torch.empty_like(d["q"])
    sel = torch.empty(w.B, w.Hkv, max(w.K - 1, 1), dtype=torch.int32, device="cuda")
    max_pages = d["page_table"].shape[1]
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, max_pages * w.block, w.d, w.K))
    binding.sas_decode_fwd_paged(d["q"], d["Kp"], d["Vp"], d["page_table"], d["seqlen"], d["s"], w.K, o, ws,
                                 w.sm_scale, sel_out=sel, apply_log_gate=apply_log_gate)
    torch.cuda.synchronize()
    return o, sel, ws


def logical_cache(pool, table, block):
    """Contiguous [B,Hkv,max_pages*block,d] copy of a paged pool (test-side torch gather)."""
    B, max_pages = table.shape
    idx = table.clamp(min=0).long()
    out = pool[idx]                                  # [B, max_pages, Hkv, block, d]
    out = out * (table >= 0).view(B, max_pages, 1, 1, 1).to(out.dtype)
    return out.permute(0, 2, 1, 3, 4).reshape(B, pool.shape[1], max_pages * block, pool.shape[3]).contiguous()


def oracle_paged(inp, w, apply_log_gate=False):
    return orc.decode_paged(to_np(inp["q"]), to_np(inp["Kp"]), to_np(inp["Vp"]), inp["page_table"].cpu().numpy(),
                            inp["seqlen"].cpu().numpy(), inp["s"].cpu().numpy().astype(np.float64), w.K, w.block,
                            w.sm_scale, apply_log_gate)


@pytest.mark.parametrize("name,B,Hq,Hkv,T,K,seqlen,gate", [
    ("g4_ragged", 5, 8, 2, 2000, 16, [2000, 1, 64, 65, 1333], False),
    ("g16_k64", 3, 16, 1, 8192, 64, [8192, 3000, 700], False),
    ("log_gate", 3, 4, 1, 1500, 5, [1500, 700, 90], True),
    ("g1_k1", 4, 2, 2, 1600, 1, [1600, 1, 129, 1000], False),
])
def test_paged_matches_oracle_and_contiguous(name, B, Hq, Hkv, T, K, seqlen, gate):
    w = workloads.custom(name, "bf16", B=B, Hq=Hq, Hkv=Hkv, d=128, T=T, K=K, decode=True)
    inp = workloads.make_paged_decode_inputs(w, seed=B + K, seqlen=seqlen)
    d = _to_dev(inp)
    o, sel, ws = run_paged(d, w, gate)
    assert binding.sas_device_status(ws) == 0
    ref_o, ref_sel = oracle_paged(inp, w, gate)
    if K > 1:
        assert np.array_equal(sel.cpu().numpy(), ref_sel)
    assert max_abs(to_np(o), ref_o) <= 2e-2
    # the contiguous call on the same logical cache: identical bits
    Kc, Vc = logical_cache(d["Kp"], d["page_table"], w.block), logical_cache(d["Vp"], d["page_table"], w.block)
    oc = torch.empty_like(o)
    selc = torch.empty_like(sel)
    wsc = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, Kc.shape[2], w.d, w.K))
    binding.sas_decode_fwd(d["q"], Kc, Vc, d["seqlen"], d["s"], w.K, oc, wsc, w.sm_scale, sel_out=selc,
                           apply_log_gate=gate)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), oc.view(torch.int16))
    if K > 1:
        assert torch.equal(sel, selc)


@pytest.mark.parametrize("name,T,B,Hq,Hkv,K,seqlen,gate", [
    ("l128k", 131072, 2, 8, 2, 16, [131072, 100001], True),     # rows of 2048 blocks: 16-warp select
    ("l512k", 524288, 1, 4, 1, 32, [524288], False),            # 8192 blocks
])
def test_paged_long_context_vs_oracle(name, T, B, Hq, Hkv, K, seqlen, gate):
    w = workloads.custom(name, "bf16", B=B, Hq=Hq, Hkv=Hkv, d=128, T=T, K=K, decode=True)
    inp = workloads.make_paged_decode_inputs(w, seed=7, seqlen=seqlen, pool_pages=64)
    o, sel, ws = run_paged(_to_dev(inp), w, gate)
    assert binding.sas_device_status(ws) == 0
    ref_o, ref_sel = oracle_paged(inp, w, gate)
    assert np.array_equal(sel.cpu().numpy(), ref_sel)
    assert max_abs(to_np(o), ref_o) <= 2e-2


@pytest.mark.parametrize("NB", [1100, 3000, 8192, 16384, 16500])
@pytest.mark.parametrize("K", [16, 64])
def test_long_row_selection_bit_exact_with_ties(NB, K):
    """Rows of 1100 to 16500 blocks (every register width of the 16-warp select, and the one-warp
    path past it), scores rounded to one decimal so that many blocks tie."""
    T = NB * 64
    w = workloads.custom("sel_long", "bf16", B=2, Hq=4, Hkv=2, d=128, T=T, K=K, decode=True)
    inp = workloads.make_paged_decode_inputs(w, seed=NB + K, seqlen=[T, T - 1000], pool_pages=8)
    inp["s"] = torch.round(inp["s"] * 10) / 10
    _, sel, ws = run_paged(_to_dev(inp), w)
    assert binding.sas_device_status(ws) == 0
    got = sel.cpu().numpy()
    s64 = inp["s"].numpy().astype(np.float64)
    for b, L in enumerate(inp["seqlen"].tolist()):
        c = (L - 1) // 64
        for g in range(w.Hkv):
            _, _, chosen = orc.topk_threshold_row(s64[b, g], c, K - 1)
            assert got[b, g].tolist() == chosen + [-1] * (K - 1 - len(chosen))


def test_paged_decode_in_a_cuda_graph():
    w = workloads.custom("graph", "bf16", B=4, Hq=8, Hkv=2, d=128, T=70000, K=16, decode=True)
    d = _to_dev(workloads.make_paged_decode_inputs(w, seed=3, seqlen=[70000, 5, 40000, 64], pool_pages=200))
    o_eager, _, _ = run_paged(d, w)
    o = torch.zeros_like(d["q"])
    max_pages = d["page_table"].shape[1]
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, max_pages * 64, w.d, w.K))
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        binding.sas_decode_fwd_paged(d["q"], d["Kp"], d["Vp"], d["page_table"], d["seqlen"], d["s"], w.K, o, ws,
                                     w.sm_scale, stream=stream)   # warm-up outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            binding.sas_decode_fwd_paged(d["q"], d["Kp"], d["Vp"], d["page_table"], d["seqlen"], d["s"], w.K, o,
                                         ws, w.sm_scale, stream=stream)
    for _ in range(2):
        o.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), o_eager.view(torch.int16))
    assert binding.sas_device_status(ws) == 0


def test_paged_page_out_of_range_is_reported():
    """A page index past the pool on an attended block: the selection kernel reports a bounds error
    and drops the block (no copy is issued for it)."""
    w = workloads.custom("badpage", "bf16", B=2, Hq=4, Hkv=1, d=128, T=1024, K=4, decode=True)
    inp = workloads.make_paged_decode_inputs(w, seed=5, seqlen=[1024, 700])
    num_pages = inp["Kp"].shape[0]
    inp["page_table"][0, (1024 - 1) // 64] = num_pages      # the current block of sequence 0
    _, _, ws = run_paged(_to_dev(inp), w)
    assert binding.sas_device_status(ws) == SAS_DEV_ERR_BOUNDS
    binding.sas_device_status_clear(ws)
    assert binding.sas_device_status(ws) == 0


def test_paged_full_size_bench_workload_sampled():
    """The bench's long-context workload as bench.py runs it (8 sequences at 524288 tokens, 69632 shuffled
    pages in an 18 GB pool, K=32): every selection list against the oracle, and the outputs of sampled
    (sequence, group) pairs against the oracle on that pair's own logical cache."""
    w = workloads.WORKLOADS["decode_b8_l512k_paged"]
    d = workloads.make_paged_decode_inputs(w, seed=0, device="cuda")
    o, sel, ws = run_paged(d, w)
    assert binding.sas_device_status(ws) == 0
    s64 = d["s"].cpu().numpy().astype(np.float64)
    got_sel = sel.cpu().numpy()
    c = (w.T - 1) // w.block
    for b in range(w.B):
        for g in range(w.Hkv):
            _, _, chosen = orc.topk_threshold_row(s64[b, g], c, w.K - 1)
            assert got_sel[b, g].tolist() == chosen
    G = w.G
    for b, g in [(0, 0), (5, 3), (7, 7)]:
        pages = d["page_table"][b].long()
        Kc = d["Kp"][pages, g].reshape(1, 1, -1, w.d)           # this group's logical cache, on the device
        Vc = d["Vp"][pages, g].reshape(1, 1, -1, w.d)
        ref, _ = orc.decode(to_np(d["q"][b:b + 1, g * G:(g + 1) * G]), to_np(Kc), to_np(Vc),
                            d["seqlen"][b:b + 1].cpu().numpy(), s64[b:b + 1, g:g + 1], w.K, w.block, w.sm_scale)
        del Kc, Vc
        assert max_abs(to_np(o[b:b + 1, g * G:(g + 1) * G]), ref) <= 2e-2
