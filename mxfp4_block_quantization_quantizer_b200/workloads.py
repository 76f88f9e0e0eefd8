"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random tensors (numpy PCG64, seeded). It holds none of
the quantizer's arithmetic; the tests, the oracle checks and the benchmark all
take their inputs from here. There is no dataset: every tensor is synthetic.

Workloads (rows x cols):
  small     256 x 512 bf16: N(0,1), 0.5% of entries x50, group (row 0,
            cols 0..31) all zero.
  deit_act  12608 x 1536 bf16: a DeiT-S MLP activation (64 images x 197
            tokens, MLP width): N(0,1) times a per-column scale drawn
            log-uniform in [0.1, 10].
  llm_w     4096 x 14336 bf16: an LLM weight: Student-t (nu = 3) x 0.02.
  osc_w     4096 x 4096 fp32 master weight ~N(0, 0.02) built so that every
            1x32 group has a known largest magnitude in [2^-4, 2^-3) and 25%
            of the other entries sit within 1e-3 relative of a rounding edge.
  sweep     8192 x 28672 bf16: N(0,1) with 0.1% of entries x100.
  master_w  4096 x 14336 fp32 LLM master weight N(0, 0.02) (Q-EMA).
"""
import numpy as np
import ml_dtypes

BF16 = ml_dtypes.bfloat16

# Shapes of the workloads, by name.
SHAPES = {
    "small": (256, 512),
    "deit_act": (12608, 1536),
    "llm_w": (4096, 14336),
    "osc_w": (4096, 4096),
    "sweep": (8192, 28672),
    "master_w": (4096, 14336),
}


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _to_bf16(a):
    """Round a float32/float64 array to bfloat16 (round to nearest even)."""
    return np.asarray(a, np.float32).astype(BF16)


def normal_bf16(rows, cols, seed, outlier_frac=0.0, outlier_scale=1.0):
    """N(0,1) bf16 with a fraction of entries multiplied by outlier_scale."""
    g = _rng(seed)
    x = g.standard_normal((rows, cols), dtype=np.float32)
    if outlier_frac > 0:
        k = max(1, int(round(outlier_frac * rows * cols)))
        idx = g.integers(0, rows * cols, size=k)
        x.reshape(-1)[idx] *= np.float32(outlier_scale)
    return _to_bf16(x)


def small(seed=0):
    x = normal_bf16(256, 512, seed, 0.005, 50.0)
    x[0, 0:32] = 0
    return x


def deit_act(seed=1, rows=12608, cols=1536):
    g = _rng(seed)
    x = g.standard_normal((rows, cols), dtype=np.float32)
    col_scale = (10.0 ** g.uniform(-1.0, 1.0, size=cols)).astype(np.float32)
    return _to_bf16(x * col_scale[None, :])


def llm_w(seed=2, rows=4096, cols=14336):
    g = _rng(seed)
    z = g.standard_normal((rows, cols), dtype=np.float32)
    chi2 = g.chisquare(3, size=(rows, cols)).astype(np.float32)
    t = z / np.sqrt(chi2 / np.float32(3.0))
    return _to_bf16(t * np.float32(0.02))


# Midpoints between neighbouring E2M1 magnitudes (0, .5, 1, 1.5, 2, 3, 4, 6):
# the inputs at which round-to-nearest changes its answer.
_EDGES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def osc_w(seed=3, rows=4096, cols=4096, edge_frac=0.25, rel=1e-3):
    """fp32 master weight for the oscillation workload.

    Every 1x32 group gets one entry of magnitude U[2^-4, 2^-3) at a random
    position and random sign; the other entries are N(0, 0.02) clipped into
    (-2^-4, 2^-4). A block scale set by the largest magnitude is therefore
    2^-6 for every group by construction. edge_frac of the other entries are
    then moved to the edge (scaled by 2^-6) nearest to them, times
    (1 + U(-rel, rel)), keeping their sign; edges at or past 2^-4 are not
    used, so no moved entry becomes the group's largest.
    """
    assert cols % 32 == 0
    g = _rng(seed)
    n_groups = rows * cols // 32
    w = g.normal(0.0, 0.02, size=(n_groups, 32))
    lim = 0.0625 * (1 - 1e-6)
    w = np.clip(w, -lim, lim)
    edges = _EDGES * 2.0 ** -6
    edges = edges[edges * (1 + rel) < lim]
    move = g.random((n_groups, 32)) < edge_frac
    mag = np.abs(w)
    hi = np.clip(np.searchsorted(edges, mag), 1, len(edges) - 1)
    lo = hi - 1
    nearest = np.where(mag - edges[lo] <= edges[hi] - mag, edges[lo], edges[hi])
    del mag, hi, lo
    jitter = 1.0 + g.uniform(-rel, rel, size=(n_groups, 32))
    w = np.where(move, np.sign(w) * nearest * jitter, w)
    top = g.uniform(0.0625, 0.125, size=n_groups)
    top_sign = np.where(g.random(n_groups) < 0.5, -1.0, 1.0)
    pos = g.integers(0, 32, size=n_groups)
    w[np.arange(n_groups), pos] = top_sign * top
    return w.astype(np.float32).reshape(rows, cols)


def master_w(seed=7, rows=4096, cols=14336):
    """fp32 master weight of an LLM linear layer: N(0, 0.02) (the Q-EMA
    workload pairs it with an EMA state drawn the same way, seed + 1)."""
    g = _rng(seed)
    return g.normal(0.0, 0.02, size=(rows, cols)).astype(np.float32)


def sweep(seed=5, rows=8192, cols=28672):
    return normal_bf16(rows, cols, seed, 0.001, 100.0)


def tensor(name, seed=None):
    """The named workload tensor (numpy, bf16 or fp32)."""
    fn = {"small": small, "deit_act": deit_act, "llm_w": llm_w,
          "osc_w": osc_w, "sweep": sweep, "master_w": master_w}[name]
    return fn() if seed is None else fn(seed)
