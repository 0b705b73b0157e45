"""Shared helpers of the parity tests: oracle-side gate preparation and error norms."""

import numpy as np
import torch

from oracle import sas_oracle as orc


def oracle_gates(s, K, block=64):
    """Oracle normalisation (fp64) and the fp32 gate tensor both sides then use.

    Returns logG64 (fp64), logG32 (fp32 numpy), tau32 (fp32), tau_idx (int32),
    sel (int32) where the selection is the oracle's on logG32.
    """
    logG64 = orc.gate_normalize(s, block)
    logG32 = logG64.astype(np.float32)
    tau, tidx, sel = orc.select_threshold(logG32.astype(np.float64), K, block)
    return logG64, logG32, tau.astype(np.float32), tidx.astype(np.int32), sel


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def dev(x, dtype=None):
    t = torch.as_tensor(x)
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().cuda()
