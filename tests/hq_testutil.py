"""Shared helpers of the GPU parity tests (CUDA path vs the fp64 oracle)."""
import numpy as np
import torch

import oracle

MAX_ABS = 2e-3      # attention outputs vs the oracle on the same quantized inputs
MEAN_ABS = 2e-4
TIE_REL = 1e-5      # index sets may differ only where oracle scores tie this closely


def to_dev(x: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    err = np.abs(np.asarray(gpu, np.float64) - ref)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max abs {mx:.3e} mean abs {mean:.3e}"
    return mx, mean


def assert_index_sets(gpu_idx: np.ndarray, ref_idx: np.ndarray, ref_score: np.ndarray,
                      window: int):
    """Sets equal except where the oracle's scores tie with its k-th score."""
    B, H, k = ref_idx.shape
    L = ref_score.shape[-1]
    n_diff = 0
    for b in range(B):
        for h in range(H):
            g, r = gpu_idx[b, h], ref_idx[b, h]
            assert np.all(np.diff(g) > 0), "GPU index list not strictly ascending"
            assert g.size == 0 or (g[0] >= 0 and g[-1] < L - window)
            if np.array_equal(g, r):
                continue
            s = ref_score[b, h]
            kth = np.sort(s[:L - window])[::-1][k - 1]
            diff = np.setxor1d(g, r)
            n_diff += diff.size
            rel = np.abs(s[diff] - kth) / max(abs(kth), 1e-300)
            assert np.all(rel <= TIE_REL), f"index sets differ beyond ties at (b={b}, h={h})"
    return n_diff


def cache_to_np(cache) -> dict:
    """The rows in use of a device cache (spare low rows left out)."""
    n = cache.n_lo
    return dict(
        k_codes=cache.k_codes[:, :, :n].cpu().numpy(), v_codes=cache.v_codes[:, :, :n].cpu().numpy(),
        k_sz=oracle.bits(cache.k_sz[:, :, :n].cpu()), v_sz=oracle.bits(cache.v_sz[:, :, :n].cpu()),
        k_hi=oracle.bits(cache.k_hi.cpu()), v_hi=oracle.bits(cache.v_hi.cpu()),
        lo_pos=cache.lo_pos[:, :, :n].cpu().numpy() if cache.lo_pos is not None else None,
        n_lo=n, n_hi=cache.n_hi, bits=cache.bits, group=cache.group,
    )


def assert_pack_equal(gpu: dict, ref: dict):
    for name in ("k_codes", "v_codes", "k_sz", "v_sz", "k_hi", "v_hi", "lo_pos"):
        if gpu.get(name) is None:
            continue
        g, r = np.asarray(gpu[name]), np.asarray(ref[name]).reshape(np.asarray(gpu[name]).shape)
        if not np.array_equal(g, r):
            bad = np.argwhere(g != r)
            raise AssertionError(f"{name}: {len(bad)} entries differ, first at {bad[0].tolist()}: "
                                 f"gpu {g[tuple(bad[0])]} oracle {r[tuple(bad[0])]}")
