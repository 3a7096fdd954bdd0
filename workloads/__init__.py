"""Seeded synthetic workloads for binarized-QK top-N attention.

This module only draws inputs: it holds none of the method's arithmetic, and
both the CUDA library's tests/benchmark and the CPU oracle take their inputs
from it.  Every tensor comes from numpy's PCG64 ``default_rng(seed)``, drawn in
fp32 in a fixed order, then rounded to bf16 (round-to-nearest-even) when the
workload is bf16.  The fp32 array handed to the oracle holds exactly the values
the device sees.

The shapes stand in for the evaluations on the source pages (HAD: GLUE/BERT at
256 tokens with top-30, ImageNet/DeiT at 197 tokens, QuALITY/T5 at 128..1024
tokens with N = 15n/128; BinaryAttention: DeiT with a learned relative-position
bias and uint8 A x int8 V, ViT at 1024x1024 = 16384 patches).  None of those
datasets is used: the values are Gaussian, with the structure described per
workload below.  "N(0, x)" means standard deviation x.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

MODE_FLOAT = 0
MODE_U8I8 = 1


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 (ties to even), returned as fp32 holding the bf16 value."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x_bf16_valued: np.ndarray) -> np.ndarray:
    """Bit pattern (uint16) of fp32 values that are already bf16-representable."""
    u = np.ascontiguousarray(x_bf16_valued, np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


@dataclass
class Bias:
    table: np.ndarray      # [H, 2gh-1, 2gw-1] fp32
    gh: int
    gw: int
    prefix: int


@dataclass
class DenseBias:
    table: np.ndarray      # [H, n, n] fp32: b_ij = table[h, i, j]


@dataclass
class Workload:
    name: str
    B: int
    H: int
    n: int
    d: int
    dtype: str             # "f32" or "bf16"
    Q: np.ndarray          # [B,H,n,d] fp32 (bf16-valued when dtype == "bf16")
    K: np.ndarray
    V: np.ndarray
    seqlens: np.ndarray | None
    bias: Bias | DenseBias | None
    passes: list           # list of (N, mode) the workload runs
    seed: int
    recipe: str
    alpha_q: np.ndarray | None = None
    alpha_k: np.ndarray | None = None
    extra: dict = field(default_factory=dict)

    @property
    def valid_tokens(self) -> int:
        if self.seqlens is None:
            return self.B * self.H * self.n
        return int(self.H * np.sum(self.seqlens))

    def valid_scores(self) -> int:
        if self.seqlens is None:
            return self.B * self.H * self.n * self.n
        return int(self.H * np.sum(self.seqlens.astype(np.int64) ** 2))


def _finish(x, dtype):
    return bf16_round(x) if dtype == "bf16" else np.ascontiguousarray(x, np.float32)


# Head dim 128 (the BinaryAttention kernel benchmark's head dim): the same recipes
# with d = 128 and seed + 100, named with a "_d128" suffix.
def _dsuf(d: int) -> str:
    return "" if d == 64 else f"_d{d}"


def _dseed(seed: int, d: int) -> int:
    return seed if d == 64 else seed + 100


def tiny(d: int = 64) -> Workload:
    """HAD-sized toy: B1 H1 n128 d64, fp32 Q,K,V iid N(0,1), seed 0; top-15 and dense, float A.V."""
    seed = _dseed(0, d)
    rng = np.random.default_rng(seed)
    shp = (1, 1, 128, d)
    Q = rng.standard_normal(shp, dtype=np.float32)
    K = rng.standard_normal(shp, dtype=np.float32)
    V = rng.standard_normal(shp, dtype=np.float32)
    return Workload("tiny_b1_h1_n128" + _dsuf(d), 1, 1, 128, d, "f32", Q, K, V, None, None,
                    [(15, MODE_FLOAT), (0, MODE_FLOAT)], seed,
                    "Q,K,V iid N(0,1) fp32; no bias; alpha=1")


def deit(d: int = 64, B: int = 64) -> Workload:
    """DeiT-shaped BinaryAttention: B64 H12 n197 (1 cls + 14x14) d64 bf16, seed 1.

    Q and K: a per-(head, channel) offset ~N(0, 0.5), shared over batch and
    tokens (one draw for Q, one for K), plus N(0,1) noise.  V: N(0,1) with
    round(0.01*H*d) = 8 of the H*d (head, channel) pairs, chosen uniformly
    without replacement, scaled x10.  Relative-position bias 27x27 per head
    ~N(0, 0.1), prefix 1 (the cls token).  Dense, uint8 A x int8 V.
    """
    seed = _dseed(1, d)
    rng = np.random.default_rng(seed)
    H, n = 12, 197
    offq = rng.standard_normal((H, d), dtype=np.float32) * np.float32(0.5)
    offk = rng.standard_normal((H, d), dtype=np.float32) * np.float32(0.5)
    Q = rng.standard_normal((B, H, n, d), dtype=np.float32) + offq[None, :, None, :]
    K = rng.standard_normal((B, H, n, d), dtype=np.float32) + offk[None, :, None, :]
    V = rng.standard_normal((B, H, n, d), dtype=np.float32)
    n_out = int(round(0.01 * H * d))
    pick = rng.choice(H * d, size=n_out, replace=False)
    for p in pick:
        V[:, p // d, :, p % d] *= np.float32(10.0)
    table = rng.standard_normal((H, 27, 27), dtype=np.float32) * np.float32(0.1)
    return Workload(f"deit_b{B}_h12_n197" + _dsuf(d), B, H, n, d, "bf16", _finish(Q, "bf16"), _finish(K, "bf16"),
                    _finish(V, "bf16"), None, Bias(table, 14, 14, 1), [(0, MODE_U8I8)], seed,
                    f"Q,K = offset[h,c]~N(0,0.5) + N(0,1); V N(0,1) with {n_out}/{H * d} channels x10; "
                    "relpos bias 27x27/head ~N(0,0.1), prefix 1",
                    extra={"outlier_channels": sorted(int(p) for p in pick)})


def deit_qkv(B: int = 64):
    """DeiT's attention inputs from their projection: X [B, 197, 768] bf16 tokens
    ~N(0,1), a random-init projection weight W [3*12*64, 768] ~N(0, 1/768) in a
    linear layer's layout (rows: Q's 768 channels, then K's, then V's), seed 9; the
    DeiT relative-position bias (27x27 per head ~N(0, 0.1), prefix 1).  Returns
    (X, W, H, bias, seqlens)."""
    rng = np.random.default_rng(9)
    H, n, Dm = 12, 197, 768
    X = _finish(rng.standard_normal((B, n, Dm), dtype=np.float32), "bf16")
    W = _finish(rng.standard_normal((3 * H * 64, Dm), dtype=np.float32) * np.float32(Dm ** -0.5), "bf16")
    table = rng.standard_normal((H, 27, 27), dtype=np.float32) * np.float32(0.1)
    return X, W, H, Bias(table, 14, 14, 1), None


def deit_dense_bias() -> Workload:
    """The DeiT workload (same Q, K, V) with a dense bias matrix instead of the
    relative-position table: one value per query-key pair, [12, 197, 197]
    ~N(0, 0.1) from seed 101.  Dense, uint8 A x int8 V."""
    w = deit()
    rng = np.random.default_rng(101)
    table = rng.standard_normal((w.H, w.n, w.n), dtype=np.float32) * np.float32(0.1)
    return Workload("deit_densebias_b64_h12_n197", w.B, w.H, w.n, w.d, w.dtype, w.Q, w.K, w.V, None,
                    DenseBias(table), [(0, MODE_U8I8)], 101,
                    w.recipe.replace("relpos bias 27x27/head ~N(0,0.1), prefix 1", "dense bias 197x197/head ~N(0,0.1)"),
                    extra=w.extra)


def bert() -> Workload:
    """BERT-shaped HAD: B32 H12 n256 d64 bf16 N(0,1), seed 2, valid lengths ~U{32..256}; top-30, float."""
    rng = np.random.default_rng(2)
    B, H, n, d = 32, 12, 256, 64
    Q = rng.standard_normal((B, H, n, d), dtype=np.float32)
    K = rng.standard_normal((B, H, n, d), dtype=np.float32)
    V = rng.standard_normal((B, H, n, d), dtype=np.float32)
    seqlens = rng.integers(32, 257, size=B).astype(np.int32)
    return Workload("bert_b32_h12_n256", B, H, n, d, "bf16", _finish(Q, "bf16"), _finish(K, "bf16"),
                    _finish(V, "bf16"), seqlens, None, [(30, MODE_FLOAT)], 2,
                    "Q,K,V iid N(0,1); L_b ~ U{32..256} per sequence; tokens past L_b are padding")


def t5(n: int, d: int = 64, B: int = 16) -> Workload:
    """T5-Base-shaped long-context sweep: B16 H12 d64 bf16, n in {128..1024}, N = 15n/128, float.

    Q ~N(0,1); K_j = 0.6 * Q_{pi(j)} + 0.8 * eps with pi(j) iid uniform over
    the n tokens of the same (b, h) and eps ~N(0,1); V ~N(0,1).  Seed 3 + log2(n/128).
    """
    assert n in (128, 256, 512, 1024)
    seed = _dseed(3 + int(np.log2(n // 128)), d)
    rng = np.random.default_rng(seed)
    H = 12
    Q = rng.standard_normal((B, H, n, d), dtype=np.float32)
    pi = rng.integers(0, n, size=(B, H, n))
    eps = rng.standard_normal((B, H, n, d), dtype=np.float32)
    K = np.float32(0.6) * np.take_along_axis(Q, pi[..., None], axis=2) + np.float32(0.8) * eps
    V = rng.standard_normal((B, H, n, d), dtype=np.float32)
    return Workload(f"t5_b{B}_h12_n{n}" + _dsuf(d), B, H, n, d, "bf16", _finish(Q, "bf16"), _finish(K, "bf16"),
                    _finish(V, "bf16"), None, None, [(15 * n // 128, MODE_FLOAT)], seed,
                    "Q N(0,1); K_j = 0.6 Q_pi(j) + 0.8 eps; V N(0,1)", extra={"pi": pi})


def stress() -> Workload:
    """Long-sequence stress: B2 H16 d64 n16384 (128x128 patches) bf16 N(0,1), seed 7.

    Relative-position bias 255x255 per head ~N(0, 0.1), prefix 0.  Two passes:
    top-1920 with float A.V, and dense with uint8 A x int8 V.
    """
    rng = np.random.default_rng(7)
    B, H, n, d = 2, 16, 16384, 64
    Q = rng.standard_normal((B, H, n, d), dtype=np.float32)
    K = rng.standard_normal((B, H, n, d), dtype=np.float32)
    V = rng.standard_normal((B, H, n, d), dtype=np.float32)
    table = rng.standard_normal((H, 255, 255), dtype=np.float32) * np.float32(0.1)
    return Workload("stress_b2_h16_n16384", B, H, n, d, "bf16", _finish(Q, "bf16"), _finish(K, "bf16"),
                    _finish(V, "bf16"), None, Bias(table, 128, 128, 0), [(1920, MODE_FLOAT), (0, MODE_U8I8)], 7,
                    "Q,K,V iid N(0,1); relpos bias 255x255/head ~N(0,0.1), prefix 0")


def grid(B: int, H: int, gh: int, gw: int, prefix: int, seqlens=None, seed: int = 11, d: int = 64) -> Workload:
    """Image-grid attention of any size: B x H heads over `prefix` class tokens
    plus a gh x gw patch grid, d64 bf16 Q,K,V iid N(0,1), a relative-position
    bias (2gh-1) x (2gw-1) per head ~N(0, 0.1), optional per-batch lengths.
    Used to cover the grid shapes the fixed workloads do not reach."""
    rng = np.random.default_rng(seed)
    n = prefix + gh * gw
    Q = rng.standard_normal((B, H, n, d), dtype=np.float32)
    K = rng.standard_normal((B, H, n, d), dtype=np.float32)
    V = rng.standard_normal((B, H, n, d), dtype=np.float32)
    table = rng.standard_normal((H, 2 * gh - 1, 2 * gw - 1), dtype=np.float32) * np.float32(0.1)
    sl = None if seqlens is None else np.asarray(seqlens, np.int32)
    return Workload(f"grid_b{B}_h{H}_{gh}x{gw}_p{prefix}" + ("" if sl is None else "_sl") + _dsuf(d), B, H, n, d, "bf16",
                    _finish(Q, "bf16"), _finish(K, "bf16"), _finish(V, "bf16"), sl, Bias(table, gh, gw, prefix),
                    [(max(1, n // 8), MODE_FLOAT), (0, MODE_U8I8)], seed,
                    "Q,K,V iid N(0,1); relpos bias ~N(0,0.1)")


def by_name(name: str) -> Workload:
    if name.endswith("_d128"):
        base = name[: -len("_d128")]
        if base == "tiny":
            return tiny(128)
        if base == "deit":
            return deit(128)
        if base.startswith("t5_"):
            return t5(int(base[3:]), 128)
        raise KeyError(name)
    if name == "tiny":
        return tiny()
    if name == "deit":
        return deit()
    if name == "bert":
        return bert()
    if name == "deit_dense_bias":
        return deit_dense_bias()
    if name.startswith("t5_"):
        return t5(int(name[3:]))
    if name == "stress":
        return stress()
    raise KeyError(name)


ALL = ["tiny", "deit", "bert", "t5_128", "t5_256", "t5_512", "t5_1024", "stress"]
