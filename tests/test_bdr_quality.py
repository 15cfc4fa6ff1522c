"""Quality of the block-diagonal Hadamard rotation (BDR) on outlier-channel inputs, measured with
the CPU oracle against unquantised fp64 attention.

SAW-INT4 (gist.science summary), section 2: a local Hadamard rotation of each block of h
dimensions spreads the energy of outlier channels before the per-token INT4 quantisation, which
is what makes token-wise INT4 usable; KV4-RL (ai.info summary), "Methodology in Plain English"
paragraph 2, stores keys in such a rotated basis.  On keys with fixed outlier channels (x15 and
x20, the synthetic workloads' recipe) the oracle's decode over the INT4 cache is compared with
fp64 attention over the unquantised inputs, for h = 1 (no rotation, "naive INT4") and h = 32, 64,
128: the logit error and the output error must both fall with the rotation.  Run with -s to see
the figures.
"""
import numpy as np
import pytest

from int4_kv_cache_append_b200 import workload as W
from oracle import oracle as O


def _errors(h: int, n_outlier: int, scale: float, seed: int = 7, s: int = 0, w: int = 0):
    lens = (700, 520, 333, 900)
    wl = W.make_workload("bdr", seed, 1, len(lens), 16, 4, 128, 16, s, w, h, lambda r: list(lens),
                         W.F32, W.F32, W.F32, n_outlier, scale)
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, wl.B)
    pool = np.zeros(O.page_bytes(cfg) * wl.num_pages, np.uint8)
    side = np.zeros(max(O.side_slot_bytes(cfg), 1) * wl.B, np.uint8)
    b = np.concatenate([np.full(L, i, np.int32) for i, L in enumerate(lens)])
    p = np.concatenate([np.arange(L, dtype=np.int32) for L in lens])
    K, V = wl.kv_inputs(0, b, p)
    O.append(cfg, pool, side, K, V, b, p, wl.lens, wl.page_table)
    q = wl.q_input(0)
    out, _ = O.decode(cfg, pool, side, q, wl.page_table, wl.lens)
    # unquantised fp64 attention on the same inputs
    ref = np.zeros_like(out)
    lerr = 0.0
    off = 0
    for i, L in enumerate(lens):
        Ki, Vi = K[off:off + L].astype(np.float64), V[off:off + L].astype(np.float64)
        off += L
        for g in range(wl.Hkv):
            kd, _, _ = O.dequant_seq(cfg, pool, side, wl.page_table[i], i, L, g)
            Hm = np.kron(np.eye(wl.D // h), _sylvester(h))
            k_unrot = kd @ Hm / h  # stored keys back in the original basis
            for j in range(g * wl.G, (g + 1) * wl.G):
                qj = q[i, j].astype(np.float64)
                lg = Ki[:, g] @ qj / np.sqrt(wl.D)
                lerr = max(lerr, float(np.abs(k_unrot @ qj / np.sqrt(wl.D) - lg).max()))
                pr = np.exp(lg - lg.max())
                ref[i, j] = (pr[:, None] * Vi[:, g]).sum(0) / pr.sum()
    d = out - ref
    return lerr, float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(ref))


def _sylvester(h: int) -> np.ndarray:
    H = np.ones((1, 1))
    while H.shape[0] < h:
        H = np.block([[H, H], [H, -H]])
    return H


@pytest.mark.parametrize("n_outlier,scale", [(4, 15.0), (2, 20.0)], ids=["4ch-x15", "2ch-x20"])
def test_rotation_cuts_the_int4_error_on_outlier_keys(n_outlier, scale):
    res = {h: _errors(h, n_outlier, scale) for h in (1, 32, 64, 128)}
    for h, (le, ma, rl) in res.items():
        print(f"outliers {n_outlier} x{scale:g}, h = {h:3d}: logit max-abs {le:.4f}, "
              f"output max-abs {ma:.4f}, output rel-L2 {rl:.5f}")
    le1, ma1, rl1 = res[1]
    for h in (32, 64, 128):
        le, ma, rl = res[h]
        assert le < 0.7 * le1, (h, le, le1)
        assert rl < rl1, (h, rl, rl1)


def test_side_cache_reduces_the_error_further():
    """With the INT8 sink/recent regions (s = 16, w = 128, the KV4-RL default) the error against
    unquantised attention is below the pure-INT4 cache's, at the same h."""
    _, _, rl_int4 = _errors(128, 4, 15.0)
    _, _, rl_side = _errors(128, 4, 15.0, s=16, w=128)
    print(f"h = 128: output rel-L2 {rl_int4:.5f} pure INT4, {rl_side:.5f} with s = 16, w = 128")
    assert rl_side < rl_int4
