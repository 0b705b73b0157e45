"""The C-ABI library loads and exports every symbol include/sas.h declares;
host-side validation and workspace sizing work without a GPU (nothing here
launches a kernel)."""

import ctypes
import os
import re

import pytest

from gated_block_sparse_flashattention_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sas.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.library_path()):
        from gated_block_sparse_flashattention_b200 import build
        build.build()
    return binding.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SAS_API\s+[\w\s\*]+?\b(sas_\w+)\s*\(", text)))


def test_header_declares_the_five_operations():
    names = declared_symbols()
    for op in ("sas_gate_normalize", "sas_select_threshold", "sas_fwd", "sas_bwd", "sas_decode_fwd"):
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 13
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(binding._SIGNATURES), "binding and header disagree"


def test_status_strings_and_version(lib):
    assert binding.status_string(0) == "SAS_OK"
    for code in (-1, -2, -3, -4, -5):
        assert binding.status_string(code).startswith("SAS_ERR")
    assert lib.sas_version() >= 100


def test_workspace_sizes(lib):
    # bf16 Qwen3-4B-like layer, K = 16: the forward keeps one partial per (position, attended block): 16 slots of
    # 4 heads x (128 bf16 + one fp32 log-sum-exp) per position and (b, g), all 8 groups in one batch
    fwd = binding.sas_fwd_workspace_size(1, 32, 8, 8192, 128, 16, binding.SAS_DT_BF16)
    bwd = binding.sas_bwd_workspace_size(1, 32, 8, 8192, 128, 16, binding.SAS_DT_BF16)
    assert fwd >= 256 + 8 * 8192 * 16 * 4 * (256 + 4)
    assert bwd >= 256 + 32 * 8192 * 4 + 32 * 8192 * 128 * 4   # Delta + fp32 dQ accumulator
    assert binding.sas_fwd_workspace_size(1, 4, 1, 1024, 64, 4, binding.SAS_DT_F32) == 256
    # partials of one (b, g) over 8 GiB (T = 256K tokens, K = 64): the q-tile union forward with its small
    # per-tile block masks (4096 q-tiles x 128 mask words) runs instead
    big = binding.sas_fwd_workspace_size(1, 4, 1, 262144, 128, 64, binding.SAS_DT_BF16)
    assert big == 256 + 8192 * 128 * 4
    # the 32K layer with K = 32 needs 1.09 GB of partials per (b, g): batches of at most 8 GiB
    c3 = binding.sas_fwd_workspace_size(2, 32, 8, 32768, 128, 32, binding.SAS_DT_BF16)
    per_group = 32768 * 32 * 4 * (256 + 4)
    assert 6 * per_group < c3 < 8 * per_group + (1 << 30)
    assert binding.sas_decode_workspace_size(16, 32, 8, 32768, 128, 16) > 0


@pytest.mark.parametrize("args,expect", [
    ((1, 32, 8, 8192, 96, binding.SAS_DT_BF16), -2),   # d = 96 not implemented
    ((1, 32, 8, 8100, 128, binding.SAS_DT_BF16), -1),  # T not a multiple of 64
    ((1, 30, 8, 8192, 128, binding.SAS_DT_BF16), -1),  # Hq not a multiple of Hkv
    ((1, 32, 8, 8192, 128, 7), -1),                    # unknown dtype
    ((1, 64, 2, 8192, 128, binding.SAS_DT_BF16), -2),  # G = 32 > 16
])
def test_workspace_size_rejects(lib, args, expect):
    out = ctypes.c_size_t(0)
    B, Hq, Hkv, T, d, dt = args
    assert lib.sas_fwd_workspace_size(B, Hq, Hkv, T, d, 64, 16, dt, ctypes.byref(out)) == expect
    assert lib.sas_fwd_workspace_size(1, 32, 8, 8192, 128, 64, 0, binding.SAS_DT_BF16, ctypes.byref(out)) == -1


def test_invalid_calls_return_errors_without_launching(lib):
    before = lib.sas_launch_count()
    fake = 0x1000  # never dereferenced: validation fails first
    assert lib.sas_gate_normalize(None, fake, 1, 1, 64, 1, 64, None) == -1
    assert lib.sas_gate_normalize(fake, fake, 1, 1, 64, 1, 64, None) == -1          # aliasing
    assert lib.sas_gate_normalize(fake, fake + 64, 1, 1, 64, 1, 32, None) == -1     # block != 64
    assert lib.sas_gate_normalize(fake + 4, fake + 64, 1, 1, 64, 1, 64, None) == -1  # misaligned
    assert lib.sas_select_threshold(fake, fake, fake, None, 1, 1, 128, 2, 64, 0, None) == -1  # K < 1
    assert lib.sas_gate_normalize_select(fake, fake + 64, fake + 128, fake + 192, None, 1, 1, 128, 2, 64, 0,
                                         None) == -1                                # K < 1
    assert lib.sas_gate_normalize_select(fake, fake, fake + 128, fake + 192, None, 1, 1, 128, 2, 64, 4,
                                         None) == -1                                # s aliases logG
    assert lib.sas_gate_normalize_select(fake, fake + 64, fake + 128, fake + 192, None, 1, 1, 192, 2, 64, 4,
                                         None) == -1                                # NB * 64 < T
    assert lib.sas_select_noisy(fake, fake + 64, fake, fake + 128, fake + 192, None, 1, 1, 128, 2, 64, 4,
                                None) == -1                                          # logG_sel aliases logG
    assert lib.sas_select_noisy(fake, fake + 64, fake + 256, fake + 128, fake + 192, None, 1, 1, 128 * 64, 2048,
                                64, 4, None) == -2                                   # rows over 1024 blocks
    def cu(*v):
        return ctypes.cast((ctypes.c_int32 * len(v))(*v), ctypes.c_void_p)
    vl = lambda c, n, T=256: lib.sas_gate_normalize_select_varlen(fake, fake + 64, fake + 128, fake + 192, None, 1,  # noqa: E731
                                                                  1, T, T // 64, 64, 4, c, n, None)
    assert vl(cu(0, 100, 256), 2) == -1          # a document not on a block boundary
    assert vl(cu(0, 128, 192), 2) == -1          # offsets end before T
    assert vl(cu(0, 128, 128, 256), 3) == -1     # an empty document
    assert vl(cu(0, 256), 0) == -1               # no document
    assert vl(cu(*range(0, 64 * 258, 64)), 257, T=64 * 257) == -2   # more than 256 documents
    assert lib.sas_gate_grad(fake, None, fake + 64, fake + 64, 1, 1, 128, 2, 64, None) == -1   # ds aliases dLogG
    assert lib.sas_gate_grad(fake, None, fake + 64, fake + 132, 1, 1, 128, 2, 64, None) == -1  # misaligned ds
    assert lib.sas_gate_grad(fake, None, fake + 64, fake + 128, 1, 1, 128, 2, 32, None) == -1  # block != 64
    assert lib.sas_gate_grad(fake, fake + 4, fake + 64, fake + 128, 1, 1, 128, 2, 64, None) == -1  # misaligned LSE
    # compact normalise + select: rows over 1024 blocks, a missing LSE output
    assert lib.sas_gate_normalize_select_compact(fake, fake + 64, fake + 128, fake + 192, None, 1, 1, 128 * 64, 2048,
                                                 64, 4, None) == -2
    assert lib.sas_gate_normalize_select_compact(fake, None, fake + 128, fake + 192, None, 1, 1, 128, 2, 64, 4,
                                                 None) == -1
    # paged decode: fp32 storage is not implemented; NBmax below max_pages is invalid
    paged = [fake] * 3 + [binding.SAS_DT_F32, fake, 4, 8, fake, fake, 4, 0, fake, None, 1, 4, 1, 4, 128, 64,
                          ctypes.c_float(0.1), fake, 1 << 20, None]
    assert lib.sas_decode_fwd_paged(*paged) == -2
    paged[3] = binding.SAS_DT_BF16
    paged[16] = 3                 # NBmax < max_pages
    assert lib.sas_decode_fwd_paged(*paged) == -1
    # sas_fwd: missing workspace / bad sizes
    args = ([fake] * 3 + [binding.SAS_DT_BF16] + [fake, None] + [fake, fake, None, fake, fake]
            + [1, 4, 1, 128, 128, 64, 2, ctypes.c_float(0.1), None, 0, None])
    assert lib.sas_fwd(*args) == -5
    args[-3] = fake
    args[-2] = 1 << 30
    args[14] = 100   # T not a multiple of 64
    assert lib.sas_fwd(*args) == -1
    args[14] = 128
    args[17] = 0     # budget K < 1
    assert lib.sas_fwd(*args) == -1
    args[17] = 2
    args[5] = fake + 4   # misaligned row LSE of compact gates
    assert lib.sas_fwd(*args) == -1
    args[5] = None
    args[8] = fake + 4   # misaligned selection index list
    assert lib.sas_fwd(*args) == -1
    assert lib.sas_launch_count() == before
