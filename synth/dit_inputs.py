"""Seeded Q/K/V for a synthetic DiT attention layer, as bf16 bit patterns.

Recipe (per (b, h) head, all draws from NumPy's PCG64 through a SeedSequence
keyed on (seed, workload id, purpose, step, tensor, head), so any single head
can be regenerated alone):

* C centroids c_1..c_C ~ N(0, I_d), each rescaled to Euclidean norm 2.
* every token n gets a label l(n) ~ Uniform{0..C-1}, shared by its Q and K.
* Q_n = 0.5*PE(t,y,x) + c_l(n) + eps,  K_n = 0.5*PE(t,y,x) + c_l(n) + eps',
  V_n ~ N(0, I_d); eps ~ N(0, 0.3^2) or 0.3 * Student-t(nu=3).
* PE is a 3D sinusoidal embedding: head_dim split into a time chunk of
  d - 2*ds and two spatial chunks of ds = 2*floor(d/6); a chunk of width w at
  position p is [sin(p*w_i), cos(p*w_i)], w_i = 10000^(-2i/w).  Tokens are
  raster ordered, time-major: n = (t*Y + y)*X + x.
* locality workloads add a*phi(pos) to both Q and K, phi being d random
  Fourier features of the Laplacian kernel exp(-|dpos|/4) on grid coordinates
  (frequencies from the 3D multivariate Cauchy of scale 1/4, uniform phases)
  and a^2 = sqrt(d), so that after the 1/sqrt(d) softmax scale a key at grid
  distance r adds about exp(-r/4) to the logit.
* denoising drift: X_s = bf16(X_{s-1} + sigma * N(0,1)), elementwise, fp32,
  independently for Q, K and V, X_{s-1} being the previous step's bf16 value.

Everything is generated in float32 and rounded to bf16 with round-to-nearest
-even; the bf16 bit patterns (uint16) are what both sides consume.
"""
from __future__ import annotations

import numpy as np

from .workloads import Workload

_PURPOSE_BASE = 0
_PURPOSE_DRIFT = 1
_PURPOSE_META = 2
_PURPOSE_BLOCKS = 3


def _rng(w: Workload, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=w.seed, spawn_key=(w.cfg_id,) + tuple(int(k) for k in key))
    return np.random.default_rng(ss)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def _bf16_to_f32(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _sincos(pos: np.ndarray, width: int) -> np.ndarray:
    half = width // 2
    i = np.arange(half, dtype=np.float64)
    omega = 10000.0 ** (-2.0 * i / width)
    ang = pos[:, None].astype(np.float64) * omega[None, :]
    return np.concatenate([np.sin(ang), np.cos(ang)], axis=1)


def _grid_positions(w: Workload):
    T, Y, X = w.grid
    n = np.arange(w.N)
    t = n // (Y * X)
    y = (n // X) % Y
    x = n % X
    return t, y, x


def position_embedding(w: Workload) -> np.ndarray:
    """[N, d] float32 3D sinusoidal embedding (time chunk first)."""
    d = w.d
    ds = 2 * (d // 6)
    dt = d - 2 * ds
    t, y, x = _grid_positions(w)
    pe = np.concatenate([_sincos(t, dt), _sincos(y, ds), _sincos(x, ds)], axis=1)
    assert pe.shape == (w.N, d)
    return pe.astype(np.float32)


def _locality_features(w: Workload, rng: np.random.Generator) -> np.ndarray:
    d = w.d
    z = rng.standard_normal((d, 3))
    g = rng.standard_normal(d)
    omega = z / (4.0 * np.abs(g)[:, None] + 1e-30)        # 3D Cauchy, scale 1/4
    phase = rng.uniform(0.0, 2.0 * np.pi, size=d)
    t, y, x = _grid_positions(w)
    pos = np.stack([t, y, x], axis=1).astype(np.float64)
    phi = np.sqrt(2.0 / d) * np.cos(pos @ omega.T + phase[None, :])
    a = d ** 0.25
    return (a * phi).astype(np.float32)


def _base_head(w: Workload, bh: int, pe: np.ndarray):
    rng = _rng(w, _PURPOSE_BASE, 0, 0, bh)
    N, d, C = w.N, w.d, w.centroids
    cent = rng.standard_normal((C, d))
    cent = 2.0 * cent / np.linalg.norm(cent, axis=1, keepdims=True)
    cent = cent.astype(np.float32)
    labels = rng.integers(0, C, size=N)
    if w.noise == "gauss":
        eq = rng.standard_normal((N, d), dtype=np.float32)
        ek = rng.standard_normal((N, d), dtype=np.float32)
    elif w.noise == "student_t3":
        eq = rng.standard_t(3, size=(N, d)).astype(np.float32)
        ek = rng.standard_t(3, size=(N, d)).astype(np.float32)
    else:
        raise ValueError(w.noise)
    v = rng.standard_normal((N, d), dtype=np.float32)
    common = 0.5 * pe + cent[labels]
    if w.locality:
        common = common + _locality_features(w, rng)
    q = common + np.float32(0.3) * eq
    k = common + np.float32(0.3) * ek
    return bf16_round(q), bf16_round(k), bf16_round(v)


def drift_head(x16: np.ndarray, w: Workload, step: int, tensor: int, bh: int) -> np.ndarray:
    """One denoising-step drift of one head's tensor (tensor: 0=Q, 1=K, 2=V)."""
    rng = _rng(w, _PURPOSE_DRIFT, step, tensor, bh)
    eps = rng.standard_normal(x16.shape, dtype=np.float32)
    return bf16_round(_bf16_to_f32(x16) + np.float32(w.drift) * eps)


def head_tensors(w: Workload, bh: int, step: int = 1, pe: np.ndarray | None = None):
    """(Q, K, V) of head bh at 1-based denoising step `step`, uint16 [N, d] each."""
    if pe is None:
        pe = position_embedding(w)
    q, k, v = _base_head(w, bh, pe)
    for s in range(2, step + 1):
        q = drift_head(q, w, s, 0, bh)
        k = drift_head(k, w, s, 1, bh)
        v = drift_head(v, w, s, 2, bh)
    return q, k, v


def layer_tensors(w: Workload, step: int = 1, heads=None):
    """(Q, K, V) uint16 [B, H, N, d] (or [len(heads), N, d] for a head subset)."""
    pe = position_embedding(w)
    sel = range(w.BH) if heads is None else list(heads)
    shape = (len(sel), w.N, w.d)
    Q = np.empty(shape, np.uint16)
    K = np.empty(shape, np.uint16)
    V = np.empty(shape, np.uint16)
    for i, bh in enumerate(sel):
        Q[i], K[i], V[i] = head_tensors(w, bh, step, pe)
    if heads is None:
        Q = Q.reshape(w.B, w.H, w.N, w.d)
        K = K.reshape(w.B, w.H, w.N, w.d)
        V = V.reshape(w.B, w.H, w.N, w.d)
    return Q, K, V


def drift_layer(X16: np.ndarray, w: Workload, step: int, tensor: int) -> np.ndarray:
    flat = X16.reshape(w.BH, w.N, w.d)
    out = np.empty_like(flat)
    for bh in range(w.BH):
        out[bh] = drift_head(flat[bh], w, step, tensor, bh)
    return out.reshape(X16.shape)


def random_metadata_head(w: Workload, bh: int, r_scale: float = 0.1):
    """Arbitrary valid metadata for one head: a random query permutation, for
    each query group k sorted unique key indices, and a random fp32 residual.

    Used to exercise the reused step on metadata of any shape without running
    a plan first.  Returns (perm int32 [N], kv_idx int32 [n_groups, k'],
    residual float32 [N, d]) with k' = min(k, N).
    """
    rng = _rng(w, _PURPOSE_META, 0, 0, bh)
    N, k = w.N, min(w.k, w.N)
    perm = rng.permutation(N).astype(np.int32)
    kv = np.empty((w.n_groups, k), np.int32)
    for g in range(w.n_groups):
        kv[g] = np.sort(rng.choice(N, size=k, replace=False)).astype(np.int32)
    res = (r_scale * rng.standard_normal((N, w.d))).astype(np.float32)
    return perm, kv, res


def random_blocks_head(w: Workload, bh: int, block: int, k_blocks: int):
    """Arbitrary valid block selections for one head: for each query group
    k_blocks sorted unique block indices in [0, N // block) (block b holds
    keys [b*block, (b+1)*block)).  Returns int32 [n_groups, k_blocks]."""
    rng = _rng(w, _PURPOSE_BLOCKS, block, k_blocks, bh)
    nb = w.N // block
    out = np.empty((w.n_groups, k_blocks), np.int32)
    for g in range(w.n_groups):
        out[g] = np.sort(rng.choice(nb, size=k_blocks, replace=False)).astype(np.int32)
    return out


def random_qkv(B: int, H: int, N: int, d: int, seed: int = 0, q_std: float = 1.0):
    """Plain Gaussian Q, K, V (bf16 bit patterns, [B, H, N, d]) for shape
    sweeps that need no DiT structure: Q ~ q_std * N(0, 1), K, V ~ N(0, 1)."""
    rng = np.random.default_rng(np.random.SeedSequence(entropy=seed, spawn_key=(99, B, H, N, d)))
    q = (q_std * rng.standard_normal((B, H, N, d))).astype(np.float32)
    k = rng.standard_normal((B, H, N, d), dtype=np.float32)
    v = rng.standard_normal((B, H, N, d), dtype=np.float32)
    return bf16_round(q), bf16_round(k), bf16_round(v)


def rising_qkv(B: int, H: int, N: int, d: int, seed: int = 0, q_std: float = 2.0, growth: float = 8.0):
    """Gaussian Q, V and keys whose scale grows with the key index,
    K_j ~ (1 + growth (j/N)^2) N(0, 1), so attention scores rise steeply along
    any ascending key list: row maxima jump by many powers of two between,
    and inside, 128-key tiles.  bf16 bit patterns [B, H, N, d]."""
    rng = np.random.default_rng(np.random.SeedSequence(entropy=seed, spawn_key=(98, B, H, N, d)))
    q = (q_std * rng.standard_normal((B, H, N, d))).astype(np.float32)
    scale = (1.0 + growth * (np.arange(N) / N) ** 2).astype(np.float32)
    k = rng.standard_normal((B, H, N, d), dtype=np.float32) * scale[:, None]
    v = rng.standard_normal((B, H, N, d), dtype=np.float32)
    return bf16_round(q), bf16_round(k), bf16_round(v)
