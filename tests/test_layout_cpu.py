"""Repository rules checked on CPU: the product path never reaches the oracle, the binding fails loudly
without the library, and the seeded input generators are deterministic and well formed."""

import pathlib
import re

import pytest
import torch

from gated_block_sparse_flashattention_b200 import binding, workloads

ROOT = pathlib.Path(__file__).resolve().parents[1]


def test_product_code_never_reaches_the_oracle():
    pkg = ROOT / "gated_block_sparse_flashattention_b200"
    files = [p for p in pkg.rglob("*") if p.suffix in {".py", ".cu", ".cuh", ".h", ".cpp"}]
    files += list((ROOT / "include").glob("*.h"))
    assert files
    for p in files:
        text = p.read_text()
        assert not re.search(r"^\s*(from|import)\s+oracle|sas_oracle|oracle/", text, re.M), p


def test_oracle_imports_nothing_of_the_product():
    for p in (ROOT / "oracle").glob("*.py"):
        text = p.read_text()
        assert "gated_block_sparse_flashattention_b200" not in text, p


def test_binding_raises_without_the_library(monkeypatch):
    monkeypatch.setattr(binding, "_LIB_PATH", str(ROOT / "no_such_library.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="not found"):
        binding.lib()


def test_generators_are_seeded_and_deterministic():
    w = workloads.custom("det", "bf16", B=1, Hq=4, Hkv=2, d=64, T=256, K=3, s_dist="normal2_planted3")
    a, b = workloads.make_training_inputs(w, seed=5), workloads.make_training_inputs(w, seed=5)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    c = workloads.make_training_inputs(w, seed=6)
    assert not torch.equal(a["Q"], c["Q"])


def test_paged_inputs_are_a_page_permutation():
    w = workloads.custom("pg", "bf16", B=3, Hq=4, Hkv=2, d=64, T=1000, K=4, decode=True)
    d = workloads.make_paged_decode_inputs(w, seed=2, seqlen=[1000, 1, 640])
    pt = d["page_table"]
    n_blocks = [(L + 63) // 64 for L in (1000, 1, 640)]
    used = torch.cat([pt[b, :n] for b, n in enumerate(n_blocks)])
    assert (used >= 0).all() and (used < d["Kp"].shape[0]).all()
    assert len(torch.unique(used)) == len(used)                     # every block its own page
    for b, n in enumerate(n_blocks):
        assert (pt[b, n:] == -1).all()
    shared = workloads.make_paged_decode_inputs(w, seed=2, seqlen=[1000, 1, 640], pool_pages=3)
    assert shared["Kp"].shape[0] == 3 and shared["page_table"].max() < 3
