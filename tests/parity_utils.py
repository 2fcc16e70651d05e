"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
binding and the CPU oracle on the same seeded inputs, and compare.

Tolerance of the fp16 output (floating point, the int8/int32 stages are
compared bit for bit): |gpu - oracle| <= 2e-3 * (1 + |oracle|) elementwise.
"""
import numpy as np
import torch

import oracle
from mixed_precision_int8_b200 import binding

RTOL = 2e-3


def assert_close_fp16(gpu: np.ndarray, ref: np.ndarray, what: str = "out"):
    g = gpu.astype(np.float64)
    r = ref.astype(np.float64)
    err = np.abs(g - r)
    lim = RTOL * (1.0 + np.abs(r))
    bad = err > lim
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at "
            f"{tuple(i)}: gpu={g[tuple(i)]} oracle={r[tuple(i)]}; "
            f"max rel err {float((err / (1 + np.abs(r))).max()):.3g}")


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_prepare(W: np.ndarray, keep_fp16: bool = False):
    Wd = to_dev(W)
    pw = binding.llmint8_prepare_weight(Wd, keep_fp16=keep_fp16)
    return pw, Wd


def gpu_matmul(X: np.ndarray, pw, alpha: float, path: int = 0,
               want_ci: bool = False, wo_build: int = 0):
    Xd = to_dev(X)
    s = X.shape[0]
    ws = binding.Workspace(s, pw.h, pw.o)
    ci = (torch.full((s, pw.o), -7, dtype=torch.int32, device="cuda")
          if want_ci else None)
    out = binding.llmint8_matmul(Xd, pw, alpha, workspace=ws, ci=ci, path=path,
                                 wo_build=wo_build)
    torch.cuda.synchronize()
    assert binding.llmint8_read_device_status(ws) == 0
    return out.cpu().numpy(), (ci.cpu().numpy() if want_ci else None), ws


def sample_rows(s: int, k: int, seed: int = 0) -> np.ndarray:
    if s <= k:
        return np.arange(s)
    rng = np.random.default_rng(seed)
    rows = set([0, s - 1, min(s - 1, 127), min(s - 1, 128)])
    rows.update(rng.choice(s, size=k - len(rows), replace=False).tolist())
    return np.array(sorted(rows))[:k]


def sample_cols(o: int, k: int, seed: int = 1) -> np.ndarray:
    if o <= k:
        return np.arange(o)
    rng = np.random.default_rng(seed)
    cols = set([0, o - 1, 255, 256, o - 16])
    cols.update(rng.choice(o, size=k - len(cols), replace=False).tolist())
    return np.array(sorted(cols))[:k]


def oracle_prepared(W: np.ndarray, cols=None):
    """Oracle Wq [nc,h] and aw for all columns or the given ones."""
    if cols is None:
        return oracle.prepare_weight(W)
    return oracle.prepare_weight(np.ascontiguousarray(W[:, cols]))


def oracle_prepared_by_blocks(W: np.ndarray, block: int = 4096):
    """Oracle Wq [o,h] and aw [o] for every column, prepared one block of
    columns at a time (each column's scale and codes depend on that column
    alone, so this is the same result with a cache-friendly footprint)."""
    parts = [oracle.prepare_weight(np.ascontiguousarray(W[:, j:j + block]))
             for j in range(0, W.shape[1], block)]
    return (np.concatenate([q for q, _ in parts]),
            np.concatenate([a for _, a in parts]))
