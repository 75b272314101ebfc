"""Seeded synthetic inputs for the SpecOPD branch-scoring pass.

Data only: this module draws random numbers and lays them out; it holds none
of the method's arithmetic (no RoPE, softmax, overlap or tree logic).  Both
the CUDA path's tests/bench and the oracle consume exactly these values.

Recipe (NumPy PCG64, seed 0 unless stated):
  * Attention inputs: trunk lengths (packed workload), anchors drawn without
    replacement from the response part of each trunk and sorted per
    sequence, then Q (branch rows), K/V (branch rows), K/V (trunk) ~ N(0,1)
    in fp32.  bf16 workloads round those fp32 draws to bf16
    (round-to-nearest-even); the GPU gets the bf16 bits and the oracle the
    identical values upcast to fp64.
  * Logits: row n of the target / draft logits is drawn from its own stream
    (seed, stream id, n), so any subset of rows can be regenerated without
    the rest.  Target row = N(0, sigma_t) plus +bump on k in {1,2,3}
    distinct uniform ids ("peaked tokens"); draft row = target row +
    N(0, sigma_d).  The overlap sweep adds 5% bit-identical rows and 5% rows
    whose draft and target have disjoint top-20 supports.
  * LM-head inputs (hidden rows and heads): target head W_t ~ N(0, (sigma /
    sqrt(d))^2), draft head W_d = W_t + N(0, (rho sigma / sqrt(d))^2); target
    hidden rows ~ N(0, 1); the draft row of position n = the target row it is
    scored against + N(0, rho^2).  So logits have spread about sigma and the
    two models agree partly.  All rounded to bf16.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Stream ids of the per-row logit generators.
_STREAM_TARGET = 11
_STREAM_DRAFT = 12
_STREAM_KIND = 13


@dataclass(frozen=True)
class AttnConfig:
    name: str
    S: int
    T: tuple            # trunk length per sequence (after drawing, for packed)
    B: int
    W: int
    Hq: int
    Hkv: int
    D: int
    dtype: str          # "f32" or "bf16"
    anchor_lo: tuple    # per sequence, inclusive
    anchor_hi: tuple    # per sequence, inclusive
    rope_base: float = 10000.0
    seed: int = 0


@dataclass(frozen=True)
class TVConfig:
    name: str
    nbranch: int
    W: int
    V: int
    dtype: str
    sigma_t: float
    sigma_d: float
    bump: float = 8.0       # +bump on 1..3 peaked ids (0 = none)
    frac_identical: float = 0.0
    frac_disjoint: float = 0.0
    seed: int = 0


def _packed_lengths(seed, S, lo, hi):
    rng = np.random.default_rng([seed, 1])
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=S))


def attn_config(name: str) -> AttnConfig:
    """The attention side of the named workload."""
    if name == "tiny":
        return AttnConfig("tiny", 1, (256,), 4, 4, 4, 1, 64, "f32", (16,), (250,))
    if name == "8b":
        return AttnConfig("8b", 1, (4096,), 64, 8, 32, 8, 128, "bf16", (2048,), (4087,))
    if name == "long":
        return AttnConfig("long", 1, (32768,), 256, 16, 40, 8, 128, "bf16",
                          (16384,), (32751,))
    if name == "packed":
        T = _packed_lengths(0, 8, 2048, 16384)
        return AttnConfig("packed", 8, T, 128, 16, 64, 8, 128, "bf16",
                          tuple(t // 2 for t in T), tuple(t - 17 for t in T))
    raise KeyError(name)


def tv_config(name: str, sigma_index: int = 0) -> TVConfig:
    """The E2E-TV side of the named workload (positions = anchors x W)."""
    if name == "tiny":
        return TVConfig("tiny", 4, 4, 1024, "f32", 2.0, 0.5, bump=0.0)
    if name == "8b":
        return TVConfig("8b", 64, 8, 151936, "bf16", 3.0, 1.0)
    if name == "sweep":
        sig = (0.0, 0.25, 1.0, 4.0)[sigma_index]
        return TVConfig(f"sweep{sigma_index}", 512, 8, 151936, "bf16", 3.0, sig,
                        frac_identical=0.05, frac_disjoint=0.05, seed=sigma_index)
    if name == "long":
        return TVConfig("long", 256, 16, 151936, "bf16", 3.0, 1.0)
    if name == "packed":
        return TVConfig("packed", 8 * 128, 16, 248320, "bf16", 3.0, 1.5)
    raise KeyError(name)


# --------------------------------------------------------------------------
# bf16 helpers (input preparation only)

def to_bf16_bits(x) -> np.ndarray:
    """Round fp32 -> bf16 bits (round to nearest, ties to even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> 16) & 1
    r = (u + np.uint32(0x7FFF) + lsb) >> 16
    # NaN stays NaN (not produced by the generators).
    return r.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x) -> np.ndarray:
    """fp32 values exactly representable in bf16 (nearest-even rounding)."""
    return bf16_bits_to_f32(to_bf16_bits(x))


# --------------------------------------------------------------------------
# Attention inputs

@dataclass
class AttnInputs:
    cfg: AttnConfig
    cu_trunk: np.ndarray   # int32 [S+1]
    anchors: np.ndarray    # int32 [S*B] local positions, sorted per sequence
    q_br: np.ndarray       # f32 [R, Hq, D]   (bf16-exact values for bf16)
    k_br: np.ndarray       # f32 [R, Hkv, D]
    v_br: np.ndarray       # f32 [R, Hkv, D]
    k_tr: np.ndarray       # f32 [T_tot, Hkv, D]  NOT rotated
    v_tr: np.ndarray       # f32 [T_tot, Hkv, D]
    extra: dict = field(default_factory=dict)

    @property
    def R(self):
        return self.q_br.shape[0]

    @property
    def T_tot(self):
        return int(self.cu_trunk[-1])


def draw_anchors(rng, S, B, lo, hi):
    out = []
    for s in range(S):
        a = rng.choice(np.arange(lo[s], hi[s] + 1), size=B, replace=False)
        out.append(np.sort(a))
    return np.concatenate(out).astype(np.int32)


def attention_inputs(cfg: AttnConfig, anchors=None) -> AttnInputs:
    rng = np.random.default_rng(cfg.seed)
    cu = np.zeros(cfg.S + 1, dtype=np.int32)
    cu[1:] = np.cumsum(cfg.T)
    if anchors is None:
        anchors = draw_anchors(rng, cfg.S, cfg.B, cfg.anchor_lo, cfg.anchor_hi)
    anchors = np.asarray(anchors, dtype=np.int32)
    R = cfg.S * cfg.B * (cfg.W - 1)
    T_tot = int(cu[-1])

    def draw(*shape):
        x = rng.standard_normal(size=shape, dtype=np.float32)
        return round_bf16(x) if cfg.dtype == "bf16" else x

    q_br = draw(R, cfg.Hq, cfg.D)
    k_br = draw(R, cfg.Hkv, cfg.D)
    v_br = draw(R, cfg.Hkv, cfg.D)
    k_tr = draw(T_tot, cfg.Hkv, cfg.D)
    v_tr = draw(T_tot, cfg.Hkv, cfg.D)
    return AttnInputs(cfg, cu, anchors, q_br, k_br, v_br, k_tr, v_tr)


def custom_attn_config(S, T, B, W, Hq, Hkv, D, dtype, anchor_lo=None, anchor_hi=None,
                       seed=0, rope_base=10000.0) -> AttnConfig:
    T = tuple(T) if isinstance(T, (tuple, list)) else (T,) * S
    lo = anchor_lo if anchor_lo is not None else tuple(0 for _ in T)
    hi = anchor_hi if anchor_hi is not None else tuple(t - 1 for t in T)
    lo = tuple(lo) if isinstance(lo, (tuple, list)) else (lo,) * S
    hi = tuple(hi) if isinstance(hi, (tuple, list)) else (hi,) * S
    return AttnConfig("custom", S, T, B, W, Hq, Hkv, D, dtype, lo, hi, rope_base, seed)


# --------------------------------------------------------------------------
# Logit rows

def _row_rng(seed, stream, n):
    return np.random.default_rng([int(seed), int(stream), int(n)])


def row_kind(cfg: TVConfig, n: int) -> str:
    """'identical', 'disjoint' or 'normal' for position n (seeded per row)."""
    if cfg.frac_identical <= 0 and cfg.frac_disjoint <= 0:
        return "normal"
    u = _row_rng(cfg.seed, _STREAM_KIND, n).random()
    if u < cfg.frac_identical:
        return "identical"
    if u < cfg.frac_identical + cfg.frac_disjoint:
        return "disjoint"
    return "normal"


def logit_rows(cfg: TVConfig, n: int):
    """(target_row, draft_row) fp32 for supervised position n (bf16-exact for
    bf16 workloads).  The target row is the row the score-row map points to
    for position n."""
    rt = _row_rng(cfg.seed, _STREAM_TARGET, n)
    zt = cfg.sigma_t * rt.standard_normal(cfg.V, dtype=np.float32)
    kind = row_kind(cfg, n)
    if kind == "disjoint":
        ids = rt.choice(cfg.V, size=40, replace=False)
        zd = zt.copy()
        zt[ids[:20]] += 24.0
        zd[ids[20:]] += 24.0
    else:
        if cfg.bump > 0:
            k = int(rt.integers(1, 4))
            ids = rt.choice(cfg.V, size=k, replace=False)
            zt[ids] += cfg.bump
        if kind == "identical":
            zd = zt.copy()
        else:
            rd = _row_rng(cfg.seed, _STREAM_DRAFT, n)
            zd = zt + cfg.sigma_d * rd.standard_normal(cfg.V, dtype=np.float32)
    if cfg.dtype == "bf16":
        zt = round_bf16(zt)
        zd = round_bf16(zd)
        if kind == "identical":
            zd = zt.copy()
    return zt.astype(np.float32), zd.astype(np.float32)


def logits(cfg: TVConfig, positions=None):
    """Stacked (z_t, z_d) fp32 [len(positions), V] for the given positions."""
    if positions is None:
        positions = range(cfg.nbranch * cfg.W)
    positions = list(positions)
    zt = np.empty((len(positions), cfg.V), dtype=np.float32)
    zd = np.empty((len(positions), cfg.V), dtype=np.float32)
    for i, n in enumerate(positions):
        zt[i], zd[i] = logit_rows(cfg, n)
    return zt, zd


# --------------------------------------------------------------------------
# LM-head inputs

@dataclass
class LmheadInputs:
    h_target: np.ndarray    # f32 [rows_target, d], bf16-exact
    target_row: np.ndarray  # int32 [N]
    w_target: np.ndarray    # f32 [V, d], bf16-exact
    h_draft: np.ndarray     # f32 [N, d], bf16-exact
    w_draft: np.ndarray     # f32 [V, d], bf16-exact


def lmhead_inputs(seed, nbranch, W, V, d, rows_target=None, sigma=3.0, rho=0.5):
    """Seeded hidden rows and LM heads (see the module recipe).  target_row is
    a random injective map of the N positions into [0, rows_target)."""
    N = nbranch * W
    rows_target = N if rows_target is None else rows_target
    rng = np.random.default_rng(seed)
    sc = sigma / np.sqrt(d)
    w_t = rng.standard_normal((V, d), dtype=np.float32) * np.float32(sc)
    w_d = w_t + rng.standard_normal((V, d), dtype=np.float32) * np.float32(rho * sc)
    h_t = rng.standard_normal((rows_target, d), dtype=np.float32)
    trow = rng.permutation(rows_target)[:N].astype(np.int32)
    h_d = h_t[trow] + rng.standard_normal((N, d), dtype=np.float32) * np.float32(rho)
    return LmheadInputs(round_bf16(h_t), trow, round_bf16(w_t), round_bf16(h_d), round_bf16(w_d))
