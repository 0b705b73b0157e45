"""The allocation-free decode entry point, sas_decode_fwd_static.

Some callers cannot allocate device memory: a plugin inside a host framework
that owns every device buffer and only hands over inputs and outputs, or a
decode loop that must not call cudaMalloc between steps. For them the library
keeps the decode step's scratch in a static device array. This test calls the
entry point through the C ABI and checks it against sas_decode_fwd (which takes
a caller workspace) and against the CPU oracle, on two calls in a row, within the
decode tolerance of the other tests, and reads the static array's status word
after each call. The file name sorts last so that a run stopping at the first
failure has already run every other test."""

import ctypes

import numpy as np
import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads
from oracle import sas_oracle as orc

pytestmark = pytest.mark.gpu


def _static_call(lib, q, Kc, Vc, seqlen, s, K, o, sel, w):
    stream = torch.cuda.current_stream().cuda_stream
    return lib.sas_decode_fwd_static(
        q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), binding.SAS_DT_BF16, seqlen.data_ptr(), s.data_ptr(), K, 0,
        o.data_ptr(), sel.data_ptr(), w.B, w.Hq, w.Hkv, w.T, w.NB, w.d, w.block, ctypes.c_float(w.sm_scale), stream)


def test_static_scratch_decode_matches_workspace_decode_twice():
    lib = binding.lib()
    w = workloads.custom("noalloc", "bf16", B=6, Hq=16, Hkv=4, d=128, T=4096, K=8, decode=True)
    for call, seed in enumerate((11, 12)):   # two calls in a row, different inputs
        inp = workloads.make_decode_inputs(w, seed=seed, seqlen=[4096, 1, 64, 65, 3000, 2049])
        q, Kc, Vc = (inp[k].cuda() for k in ("q", "Kc", "Vc"))
        s, seqlen = inp["s"].cuda(), inp["seqlen"].cuda()
        o_ref = torch.empty_like(q)
        sel_ref = torch.empty(w.B, w.Hkv, w.K - 1, dtype=torch.int32, device="cuda")
        ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K))
        binding.sas_decode_fwd(q, Kc, Vc, seqlen, s, w.K, o_ref, ws, w.sm_scale, sel_out=sel_ref)
        o = torch.full_like(q, float("nan"))
        sel = torch.full_like(sel_ref, -7)
        assert _static_call(lib, q, Kc, Vc, seqlen, s, w.K, o, sel, w) == 0
        torch.cuda.synchronize()
        assert binding.sas_decode_static_status() == 0, f"call {call}: kernel-side error"
        assert torch.equal(sel, sel_ref), f"call {call}: selected blocks differ"
        err = (o.float() - o_ref.float()).abs().max().item()
        assert err <= 2e-2, f"call {call}: max-abs difference {err}"
        f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
        ref_o, ref_sel = orc.decode(f64(inp["q"]), f64(inp["Kc"]), f64(inp["Vc"]), inp["seqlen"].numpy(),
                                    inp["s"].numpy().astype(np.float64), w.K, w.block, w.sm_scale)
        assert np.array_equal(sel.cpu().numpy(), ref_sel), f"call {call}: selection differs from the oracle"
        err_o = np.abs(o.float().cpu().numpy() - ref_o).max()
        assert err_o <= 2e-2, f"call {call}: max-abs difference {err_o} against the oracle"


def test_static_scratch_rejects_problems_beyond_its_limit():
    lib = binding.lib()
    # 512 (batch, KV group) pairs x 32 splits x 8 heads x 128 features of fp32 partials: > 8 MiB.
    fake = 0x1000   # never dereferenced: the size check fails first
    st = lib.sas_decode_fwd_static(fake, fake, fake, binding.SAS_DT_BF16, fake, fake, 64, 0, fake, None,
                                   64, 64, 8, 4096, 64, 128, 64, ctypes.c_float(0.1), None)
    assert st == -5
