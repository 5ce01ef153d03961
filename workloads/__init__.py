"""Seeded synthetic inputs for the HSTU attention hot path.

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no bucket function, no SiLU, no masking, no attention):
both the fp64 oracle under ``oracle/`` and the CUDA path receive exactly the
arrays built here.

Workloads (shapes follow the HSTU benchmark described on "Déploiement de
recommandeurs génératifs avec NVIDIA Dynamo-Triton et HSTU", section "Détails
clés": hidden 512, 4 heads, bf16, histories up to 8192 tokens; the public
KuaiRand-1K data named there is not available, so these synthetic draws stand
in for it):

* ``tiny_fp32``       B=2, L={17,40}, H=2, d=32, fp32, 16-bucket position rab, N=40
* ``jagged_bf16``     B=8, L~U[256,2048], H=4, d=128, bf16, 128-bucket position
                      + 64-bucket time-gap rab, timestamps with Exp(300 s) gaps,
                      scale 1/max_len
* ``cached_cand``     B=8, cached history L~U[1024,4096] in 32-token pages with a
                      shuffled free list, +64 appended tokens, 128 candidates/user
* ``block_stack``     B=8, L~U[512,4096], d_model 512, 8 layers, W~N(0,0.02)
* ``long_history``    B=32, L=clip(zipf(1.2),64,16384), pool of 2M tokens,
                      16 appended tokens per user, causal attention over all L

Each workload ``k`` (1..5 in the order above) draws from
``numpy.random.default_rng(1000 + k)`` in a fixed order: lengths, timestamps,
rab tables, Q, K, V, appended / candidate tensors, weights, page free order.

Floating-point tensors are returned as numpy float32 arrays holding values that
are exactly representable in the stated storage dtype (bf16 values are rounded
once, here, by torch's RNE conversion).  ``to_torch`` gives the storage-dtype
torch tensors that the CUDA path consumes; the oracle upcasts the same values.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

TS0 = 1_700_000_000          # first timestamp of every user (seconds)
GAP_MEAN_S = 300.0           # mean of the exponential inter-event gap
PAGE = 32                    # tokens per KV page


def _as_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 draws to the storage dtype (values stay float32 arrays)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        import torch
        return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


def to_torch(x: np.ndarray, dtype: str):
    """Storage-dtype torch CPU tensor for a float array from this module."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t.clone()


def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off


def draw_timestamps(rng: np.random.Generator, lengths, gap_mean: float = GAP_MEAN_S,
                    kind: str = "increasing") -> np.ndarray:
    """int64 timestamps per user, starting at TS0.

    kind "increasing": gaps 1 + floor(Exp(gap_mean)), strictly increasing (the
    workloads' recipe; gap_mean of days gives spans of years).
    kind "unordered": gaps uniform in [-gap_mean, gap_mean], so neighbours may be
    equal or decreasing (logs merged from several sources)."""
    if kind not in ("increasing", "unordered"):
        raise ValueError(kind)
    out = []
    for L in lengths:
        if kind == "increasing":
            gaps = 1 + np.floor(rng.exponential(gap_mean, size=int(L) - 1)).astype(np.int64)
        else:
            g = int(gap_mean)
            gaps = rng.integers(-g, g, size=int(L) - 1, endpoint=True).astype(np.int64)
        ts = np.empty(int(L), dtype=np.int64)
        ts[0] = TS0
        if L > 1:
            ts[1:] = TS0 + np.cumsum(gaps)
        out.append(ts)
    return np.concatenate(out) if out else np.zeros(0, np.int64)


@dataclasses.dataclass
class JaggedCase:
    """Self-attention over jagged sequences (causal)."""
    name: str
    dtype: str                       # "f32" | "bf16"
    lengths: np.ndarray              # [B] int64
    seq_offsets: np.ndarray          # [B+1] int64
    H: int
    d: int
    q: np.ndarray                    # [T,H,d] float32 (storage-exact)
    k: np.ndarray
    v: np.ndarray
    pos_table: np.ndarray            # [n_pos] float32
    time_table: Optional[np.ndarray]  # [n_time] float32 or None
    timestamps: Optional[np.ndarray]  # [T] int64 or None
    scale: float

    @property
    def B(self):
        return len(self.lengths)

    @property
    def T(self):
        return int(self.seq_offsets[-1])

    @property
    def max_len(self):
        return int(self.lengths.max()) if len(self.lengths) else 0

    def flops(self) -> float:
        """Algorithmic flops: unmasked pairs x (2 d_qk + 2 d_v) x H."""
        L = self.lengths.astype(np.float64)
        return float((L * (L + 1) / 2).sum() * self.H * 4 * self.d)


def jagged_case(seed: int, lengths, H: int, d: int, dtype: str = "bf16",
                n_pos: int = 16, n_time: int = 0, scale: Optional[float] = None,
                name: str = "custom", rng: Optional[np.random.Generator] = None,
                ts_gap_mean: float = GAP_MEAN_S, ts_kind: str = "increasing") -> JaggedCase:
    """Build a jagged causal case with given lengths (rab tables ~ N(0, 0.1))."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    off = offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = draw_timestamps(rng, lengths, ts_gap_mean, ts_kind) if n_time > 0 else None
    pos_table = rng.normal(0.0, 0.1, size=n_pos).astype(np.float32)
    time_table = rng.normal(0.0, 0.1, size=n_time).astype(np.float32) if n_time > 0 else None
    q = _as_storage(rng.standard_normal((T, H, d), dtype=np.float32), dtype)
    k = _as_storage(rng.standard_normal((T, H, d), dtype=np.float32), dtype)
    v = _as_storage(rng.standard_normal((T, H, d), dtype=np.float32), dtype)
    if scale is None:
        scale = 1.0 / max(int(lengths.max()) if len(lengths) else 1, 1)
    return JaggedCase(name, dtype, lengths, off, H, d, q, k, v, pos_table, time_table, ts, float(scale))


def tiny_fp32() -> JaggedCase:
    """Workload 1: B=2, L={17,40}, H=2, d=32, fp32, 16 position buckets, N=40."""
    return jagged_case(1001, [17, 40], H=2, d=32, dtype="f32", n_pos=16, n_time=0,
                       scale=1.0 / 40.0, name="tiny_fp32")


def jagged_bf16(B: int = 8, lmin: int = 256, lmax: int = 2048) -> JaggedCase:
    """Workload 2: B=8, L~U[256,2048], H=4, d=128, bf16, pos(128)+time(64) rab, 1/max_len."""
    rng = np.random.default_rng(1002)
    lengths = rng.integers(lmin, lmax, size=B, endpoint=True).astype(np.int64)
    return jagged_case(1002, lengths, H=4, d=128, dtype="bf16", n_pos=128, n_time=64,
                       scale=None, name="jagged_bf16", rng=rng)


@dataclasses.dataclass
class CachedCase:
    """Paged-KV workloads: a pre-filled history, an appended delta, then queries."""
    name: str
    H: int
    d: int
    hist_lengths: np.ndarray         # [B] tokens already cached before the step
    n_new: np.ndarray                # [B] tokens appended during the step
    hist_k: np.ndarray               # [sum hist, H, d]
    hist_v: np.ndarray
    new_k: np.ndarray                # [sum n_new, H, d]
    new_v: np.ndarray
    pos_table: np.ndarray
    n_pages: int
    free_order: np.ndarray           # [n_pages] int32 permutation (stack; top = last)
    mode: int                        # 0: candidates see history+self; 1: causal suffix
    # mode 0
    n_cand: Optional[np.ndarray] = None
    q_cand: Optional[np.ndarray] = None
    k_cand: Optional[np.ndarray] = None
    v_cand: Optional[np.ndarray] = None
    # mode 1: queries are the last n_q tokens of each cached sequence
    q: Optional[np.ndarray] = None
    n_q: Optional[np.ndarray] = None
    scale: float = 1.0

    @property
    def B(self):
        return len(self.hist_lengths)

    @property
    def users(self) -> np.ndarray:
        return np.arange(self.B, dtype=np.int64)

    @property
    def total_lengths(self) -> np.ndarray:
        return self.hist_lengths + self.n_new

    @property
    def q_offsets(self) -> np.ndarray:
        return offsets_from_lengths(self.n_cand if self.mode == 0 else self.n_q)

    def flops(self) -> float:
        Lk = self.total_lengths.astype(np.float64)
        if self.mode == 0:
            pairs = (self.n_cand * (Lk + 1)).sum()
        else:
            nq = self.n_q.astype(np.float64)
            pairs = (nq * (Lk - nq) + nq * (nq + 1) / 2).sum()
        return float(pairs * self.H * 4 * self.d)

    def algorithmic_bytes(self) -> float:
        """Minimum HBM bytes of one step (append + cached attention)."""
        row = self.H * self.d * 2
        Lk = self.total_lengths.astype(np.float64)
        kv_read = (Lk * 2 * row).sum()
        append = (self.n_new.astype(np.float64) * 2 * row * 2).sum()
        nq = (self.n_cand if self.mode == 0 else self.n_q).astype(np.float64).sum()
        io = nq * row * (4 if self.mode == 0 else 2)
        return float(kv_read + append + io)


def cached_cand(B: int = 8, hmin: int = 1024, hmax: int = 4096, n_new: int = 64,
                n_cand: int = 128, seed: int = 1003, slack: float = 1.25) -> CachedCase:
    """Workload 3: candidates scored against a paged history (100% KV hit)."""
    rng = np.random.default_rng(seed)
    H, d = 4, 128
    hist = rng.integers(hmin, hmax, size=B, endpoint=True).astype(np.int64)
    pos_table = rng.normal(0.0, 0.1, size=16).astype(np.float32)
    Th, Tn, Tc = int(hist.sum()), B * n_new, B * n_cand
    hist_k = _as_storage(rng.standard_normal((Th, H, d), dtype=np.float32), "bf16")
    hist_v = _as_storage(rng.standard_normal((Th, H, d), dtype=np.float32), "bf16")
    new_k = _as_storage(rng.standard_normal((Tn, H, d), dtype=np.float32), "bf16")
    new_v = _as_storage(rng.standard_normal((Tn, H, d), dtype=np.float32), "bf16")
    q_c = _as_storage(rng.standard_normal((Tc, H, d), dtype=np.float32), "bf16")
    k_c = _as_storage(rng.standard_normal((Tc, H, d), dtype=np.float32), "bf16")
    v_c = _as_storage(rng.standard_normal((Tc, H, d), dtype=np.float32), "bf16")
    need = int(np.sum((hist + n_new + PAGE - 1) // PAGE))
    n_pages = int(np.ceil(need * slack))
    free_order = rng.permutation(n_pages).astype(np.int32)
    N = int((hist + n_new + n_cand).max())
    return CachedCase("cached_cand", H, d, hist, np.full(B, n_new, np.int64), hist_k, hist_v,
                      new_k, new_v, pos_table, n_pages, free_order, mode=0,
                      n_cand=np.full(B, n_cand, np.int64), q_cand=q_c, k_cand=k_c, v_cand=v_c,
                      scale=1.0 / N)


def long_history(B: int = 32, lmin: int = 64, lmax: int = 16384, n_new: int = 16,
                 pool_tokens: int = 2 * 1024 * 1024, seed: int = 1005,
                 lengths=None) -> CachedCase:
    """Workload 5: Zipf(1.2) lengths clipped to [64,16384]; causal over the full history."""
    rng = np.random.default_rng(seed)
    H, d = 4, 128
    if lengths is None:
        L = np.clip(rng.zipf(1.2, size=B), lmin, lmax).astype(np.int64)
    else:
        L = np.asarray(lengths, dtype=np.int64)
    pos_table = rng.normal(0.0, 0.1, size=16).astype(np.float32)
    nn_ = np.minimum(np.full(len(L), n_new, np.int64), L)
    hist = L - nn_
    T = int(L.sum())
    # Q, K, V for all L tokens of every user; the last n_new K/V rows of each user
    # are the appended delta, the rest is the pre-filled history.
    q = _as_storage(rng.standard_normal((T, H, d), dtype=np.float32), "bf16")
    k = _as_storage(rng.standard_normal((T, H, d), dtype=np.float32), "bf16")
    v = _as_storage(rng.standard_normal((T, H, d), dtype=np.float32), "bf16")
    off = offsets_from_lengths(L)
    hk, hv, nk, nv = [], [], [], []
    for b in range(len(L)):
        s, e = int(off[b]), int(off[b + 1])
        hk.append(k[s:e - nn_[b]]); hv.append(v[s:e - nn_[b]])
        nk.append(k[e - nn_[b]:e]); nv.append(v[e - nn_[b]:e])
    n_pages = max(pool_tokens // PAGE, int(np.sum((L + PAGE - 1) // PAGE)))
    free_order = rng.permutation(n_pages).astype(np.int32)
    return CachedCase("long_history", H, d, hist, nn_, np.concatenate(hk), np.concatenate(hv),
                      np.concatenate(nk), np.concatenate(nv), pos_table, n_pages, free_order,
                      mode=1, q=q, n_q=L.copy(), scale=1.0 / int(L.max()))


@dataclasses.dataclass
class BlockCase:
    """HSTU block stack: X -> SiLU(X W1) = [U|V|Q|K] -> attention -> LN(A)*U -> X + G W2."""
    name: str
    lengths: np.ndarray
    seq_offsets: np.ndarray
    d_model: int
    H: int
    dh: int
    n_layers: int
    x0: np.ndarray                   # [T, d_model] bf16-exact
    w_uvqk: np.ndarray               # [n_layers, d_model, 4*H*dh] bf16-exact
    w_o: np.ndarray                  # [n_layers, H*dh, d_model] bf16-exact
    pos_table: np.ndarray
    time_table: np.ndarray
    timestamps: np.ndarray
    scale: float
    ln_eps: float = 1e-5

    @property
    def B(self):
        return len(self.lengths)

    @property
    def T(self):
        return int(self.seq_offsets[-1])

    def flops(self) -> float:
        T = float(self.T)
        gemm = 2 * T * self.d_model * (4 * self.H * self.dh) + 2 * T * (self.H * self.dh) * self.d_model
        L = self.lengths.astype(np.float64)
        attn = (L * (L + 1) / 2).sum() * self.H * 4 * self.dh
        return float(self.n_layers * (gemm + attn))


def block_case(seed: int, lengths, n_layers: int, d_model: int = 512, H: int = 4, dh: int = 128,
               rng: Optional[np.random.Generator] = None, name: str = "custom",
               n_pos: int = 128, n_time: int = 64, ts_gap_mean: float = GAP_MEAN_S,
               ts_kind: str = "increasing") -> BlockCase:
    rng = rng if rng is not None else np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    off = offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = draw_timestamps(rng, lengths, ts_gap_mean, ts_kind)
    pos_table = rng.normal(0.0, 0.1, size=n_pos).astype(np.float32)
    time_table = rng.normal(0.0, 0.1, size=n_time).astype(np.float32)
    x0 = _as_storage(rng.standard_normal((T, d_model), dtype=np.float32), "bf16")
    w1 = _as_storage(rng.normal(0.0, 0.02, size=(n_layers, d_model, 4 * H * dh)).astype(np.float32), "bf16")
    w2 = _as_storage(rng.normal(0.0, 0.02, size=(n_layers, H * dh, d_model)).astype(np.float32), "bf16")
    return BlockCase(name, lengths, off, d_model, H, dh, n_layers, x0, w1, w2, pos_table,
                     time_table, ts, 1.0 / int(lengths.max()))


def block_stack(B: int = 8, lmin: int = 512, lmax: int = 4096, n_layers: int = 8) -> BlockCase:
    """Workload 4: 8-layer HSTU block stack, d_model 512, 4 heads x 128."""
    rng = np.random.default_rng(1004)
    lengths = rng.integers(lmin, lmax, size=B, endpoint=True).astype(np.int64)
    return block_case(1004, lengths, n_layers, rng=rng, name="block_stack")
