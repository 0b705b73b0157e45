"""The one-kernel bf16 decode step (one CTA per (b, g)) against the oracle.

A contiguous bf16 cache whose score rows have at most 512 blocks, with at least
three (b, g) groups per four SMs, runs the whole step as decode_group_kernel:
each CTA selects its group's blocks, streams them and writes o. Up to one group
per SM it keeps six ring stages, beyond that three (two CTAs per SM). Checked
here on both: the selection bit-exact, o within 2e-2 max-abs of the oracle, one
kernel launch per call, and the same bits when the call is repeated (the warps'
states are combined in a fixed order)."""

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc
from tests.helpers import dev, max_abs, to_np

pytestmark = pytest.mark.gpu


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


CASES = [
    # name, B, Hq, Hkv, T, K, sequence lengths (repeated over the batch), log gate
    ("g4_ragged", 32, 16, 4, 2000, 16, [2000, 1, 64, 65, 1333, 128, 129, 1999], False),
    ("g16_every_block", 128, 16, 1, 1600, 40, [1600, 1, 129, 1000], False),
    ("g5_k64", 64, 10, 2, 8192, 64, [8192, 3000, 700, 64], False),
    ("g4_k1", 32, 16, 4, 2000, 1, [2000, 1, 65, 777], False),
    ("g1_k2", 128, 1, 1, 3000, 2, [3000, 2999, 65, 1], False),
    ("log_gate", 120, 4, 1, 1500, 5, [1500, 700, 90, 1], True),
    ("rows_of_257_blocks", 112, 4, 1, 16448, 16, [16448, 16385, 1025, 64], False),
    ("three_stages", 40, 32, 8, 4096, 16, [4096, 2000, 1, 4095, 3000], False),
]


@pytest.mark.parametrize("name,B,Hq,Hkv,T,K,lengths,gate", CASES, ids=[c[0] for c in CASES])
def test_group_decode_matches_oracle(name, B, Hq, Hkv, T, K, lengths, gate):
    assert 4 * B * Hkv >= 3 * _sms(), "the case must reach the one-kernel path"
    w = workloads.custom(name, "bf16", B=B, Hq=Hq, Hkv=Hkv, d=128, T=T, K=K, decode=True)
    seqlen = (lengths * ((B + len(lengths) - 1) // len(lengths)))[:B]
    inp = workloads.make_decode_inputs(w, seed=B + K, seqlen=seqlen)
    q, Kc, Vc, s, sl = (dev(inp[k]) for k in ("q", "Kc", "Vc", "s", "seqlen"))
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K))
    outs = []
    for _ in range(2):
        o = torch.empty_like(q)
        sel = torch.empty(w.B, w.Hkv, max(w.K - 1, 1), dtype=torch.int32, device="cuda")
        n0 = binding.launch_count()
        binding.sas_decode_fwd(q, Kc, Vc, sl, s, w.K, o, ws, w.sm_scale, sel_out=sel, apply_log_gate=gate)
        launches = binding.launch_count() - n0
        torch.cuda.synchronize()
        assert binding.sas_device_status(ws) == 0
        assert launches == 1, launches
        outs.append((o, sel))
    (o, sel), (o2, sel2) = outs
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16))
    if w.K > 1:
        assert torch.equal(sel, sel2)
    ref_o, ref_sel = orc.decode(to_np(inp["q"]), to_np(inp["Kc"]), to_np(inp["Vc"]), inp["seqlen"].numpy(),
                                inp["s"].numpy().astype(np.float64), w.K, w.block, w.sm_scale, gate)
    if w.K > 1:
        assert np.array_equal(sel.cpu().numpy(), ref_sel)
    assert max_abs(to_np(o), ref_o) <= 2e-2, max_abs(to_np(o), ref_o)


def test_group_decode_without_sel_out():
    """Without sel_out the selection keeps its (key, index) order for the attended list: same o within
    rounding of the order of the blocks."""
    w = workloads.custom("no_sel", "bf16", B=32, Hq=16, Hkv=4, d=128, T=4096, K=12, decode=True)
    inp = workloads.make_decode_inputs(w, seed=3, seqlen=([4096, 3000, 1500, 100] * 8))
    q, Kc, Vc, s, sl = (dev(inp[k]) for k in ("q", "Kc", "Vc", "s", "seqlen"))
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K))
    o = torch.empty_like(q)
    binding.sas_decode_fwd(q, Kc, Vc, sl, s, w.K, o, ws, w.sm_scale)
    torch.cuda.synchronize()
    assert binding.sas_device_status(ws) == 0
    ref_o, _ = orc.decode(to_np(inp["q"]), to_np(inp["Kc"]), to_np(inp["Vc"]), inp["seqlen"].numpy(),
                          inp["s"].numpy().astype(np.float64), w.K, w.block, w.sm_scale, False)
    assert max_abs(to_np(o), ref_o) <= 2e-2


def test_group_decode_length_outside_the_cache_is_reported():
    """A sequence length of 0 (or past the cache) is a bounds error in the status word; the call completes."""
    w = workloads.custom("bad_len", "bf16", B=32, Hq=16, Hkv=4, d=128, T=1024, K=4, decode=True)
    inp = workloads.make_decode_inputs(w, seed=5, seqlen=[1024, 0] + [500] * 30)
    q, Kc, Vc, s, sl = (dev(inp[k]) for k in ("q", "Kc", "Vc", "s", "seqlen"))
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K))
    o = torch.empty_like(q)
    binding.sas_decode_fwd(q, Kc, Vc, sl, s, w.K, o, ws, w.sm_scale)
    torch.cuda.synchronize()
    assert binding.sas_device_status(ws) == 2
