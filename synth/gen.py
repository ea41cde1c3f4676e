"""Host (NumPy) implementation of the synthetic input recipes.

Recipe (one definition, implemented here and in synth/csrc/synth.cu):

* Counter-based draws: Philox4x32-10 (Salmon et al., SC'11; own copy), key =
  seed, counter = (position // 4, row id, sub-stream, 7), word = position % 4.
  Sub-streams: 0 target noise, 1 draft noise, 2 head rotation, 3 head offsets,
  4 draft-token Gumbel noise.
* Standard normal from one 32-bit word w: piecewise-linear inverse CDF over a
  4097-entry table T[j] = Phi^-1((j + 1/2) / 4097):  i = w >> 20,
  f = (w & 0xFFFFF) * 2^-20,  n = T[i] + (T[i+1] - T[i]) * f  (fp32, each
  operation rounded on its own).  Tails are cut near +-3.7 sigma.
* Target row r:  zT_v = sigma_z * n_v, then a Zipf(1.1) head: V is split into
  L blocks of V // L entries; block j holds one head token at a random offset;
  ranks are assigned by a random rotation; zT[h] += beta * rank^-1.1 with
  beta = ln V + sigma_z^2 / 2 + 2 (an LM-like peak: at tau = 1 the rank-1 token
  carries most of the mass).  Stored as bf16 (round to nearest even) or fp32.
* Draft row paired with target row r:  zD_v = zT_v + sigma_d * n'_v (from the
  fp32 target value before rounding), stored like the target.
* Draft token for a draft row: a stand-in for the drafter's own sampler,
  x = argmax_v (zD_v * (1/tau) + G_v) with G_v = -ln(-ln u_v), u_v 23-bit
  uniform, and ln a fixed fp32 routine (range reduction to [sqrt(1/2),
  sqrt(2)) and the atanh series ln m = 2 (s + s^3/3 + ... + s^9/9),
  s = (m - 1)/(m + 1)) written with plain rounded operations so host and
  device agree bit for bit.  Ties go to the lower index.
* Page tables, sparse top-10 rows: host only (small), from integer maps and
  numpy's default_rng.
"""

from dataclasses import dataclass, field

import numpy as np
from scipy import special

_MASK = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)
TAG = 7
SUB_TARGET, SUB_DRAFT, SUB_ROT, SUB_HEAD, SUB_DRAFT_TOKEN = 0, 1, 2, 3, 4
F32 = np.float32


def _philox(c0, c1, c2, c3, k0, k1):
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK for c in (c0, c1, c2, c3))
    k0 = np.uint64(k0)
    k1 = np.uint64(k1)
    for rnd in range(10):
        p0 = np.uint64(0xD2511F53) * c0
        p1 = np.uint64(0xCD9E8D57) * c2
        c0, c1, c2, c3 = ((p1 >> _S32) ^ c1 ^ k0, p1 & _MASK, (p0 >> _S32) ^ c3 ^ k1, p0 & _MASK)
        if rnd != 9:
            k0 = (k0 + np.uint64(0x9E3779B9)) & _MASK
            k1 = (k1 + np.uint64(0xBB67AE85)) & _MASK
    return c0, c1, c2, c3


def words(seed, row_ids, sub, n):
    """[R, n] uint64 holding 32-bit words for positions 0..n-1 of each row id."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    rows = np.asarray(row_ids, dtype=np.uint64).reshape(-1)
    ncall = (int(n) + 3) // 4
    c0 = np.arange(ncall, dtype=np.uint64)
    out = _philox(c0[None, :], rows[:, None], sub, TAG, seed & 0xFFFFFFFF, seed >> 32)
    return np.stack(out, axis=-1).reshape(rows.shape[0], -1)[:, :n]


def normal_table():
    j = np.arange(4097, dtype=np.float64)
    return special.ndtri((j + 0.5) / 4097.0).astype(F32)


_TABLE = None


def _table():
    global _TABLE
    if _TABLE is None:
        _TABLE = normal_table()
    return _TABLE


def normals(w):
    T = _table()
    w = np.asarray(w, dtype=np.uint64)
    i = (w >> np.uint64(20)).astype(np.int64)
    f = (w & np.uint64(0xFFFFF)).astype(F32) * F32(2.0 ** -20)
    t0 = T[i]
    d = T[i + 1] - t0
    return t0 + d * f


def head_boosts(L, sigma_z, V):
    beta = np.log(float(V)) + float(sigma_z) ** 2 / 2.0 + 2.0
    return (beta * np.arange(1, L + 1, dtype=np.float64) ** -1.1).astype(F32)


def head_positions(seed, row_ids, V, L):
    """Head token ids [R, L] and their Zipf ranks (0-based) [R, L]."""
    bs = V // L
    rot = (words(seed, row_ids, SUB_ROT, 1)[:, 0] % np.uint64(L)).astype(np.int64)
    offs = (words(seed, row_ids, SUB_HEAD, L) % np.uint64(bs)).astype(np.int64)
    pos = np.arange(L, dtype=np.int64)[None, :] * bs + offs
    rank = (np.arange(L, dtype=np.int64)[None, :] + rot[:, None]) % L
    return pos, rank


def f32_to_bf16_bits(x):
    b = np.asarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b):
    return (np.asarray(b, dtype=np.uint32) << np.uint32(16)).view(F32)


def gen_rows(seed, row_ids, V, sigma_z, L, sigma_d=None, dtype="bf16", want_target=True):
    """Target rows (and paired draft rows if sigma_d is given) for the given row ids.

    Returns (zT, zD) as float32 arrays holding the stored values (bf16 values
    are exact in fp32); zD is None without sigma_d.  ``want_target=False``
    skips returning the target (it is still computed: the draft depends on it).
    """
    rows = np.asarray(row_ids, dtype=np.int64).reshape(-1)
    zt = F32(sigma_z) * normals(words(seed, rows, SUB_TARGET, V))
    if L > 0:
        pos, rank = head_positions(seed, rows, V, L)
        boosts = head_boosts(L, sigma_z, V)
        ridx = np.arange(rows.shape[0])[:, None]
        zt[ridx, pos] = zt[ridx, pos] + boosts[rank]
    zd = None
    if sigma_d is not None:
        sd = np.broadcast_to(np.asarray(sigma_d, dtype=F32), rows.shape)
        zd = zt + sd[:, None] * normals(words(seed, rows, SUB_DRAFT, V))
    if dtype == "bf16":
        zt_s = bf16_bits_to_f32(f32_to_bf16_bits(zt)) if want_target else None
        zd_s = None if zd is None else bf16_bits_to_f32(f32_to_bf16_bits(zd))
    else:
        zt_s = zt if want_target else None
        zd_s = zd
    return zt_s, zd_s


_SQRT2 = F32(1.41421356)
_LN2 = F32(np.log(2.0))
_C = [F32(2.0), F32(2.0 / 3.0), F32(2.0 / 5.0), F32(2.0 / 7.0), F32(2.0 / 9.0)]


def synth_log(x):
    """ln x for normal positive fp32 x with plain rounded fp32 operations."""
    x = np.asarray(x, dtype=F32)
    bits = x.view(np.uint32)
    e = (bits >> np.uint32(23)).astype(np.int32) - 127
    m = ((bits & np.uint32(0x7FFFFF)) | np.uint32(0x3F800000)).view(F32)
    big = m > _SQRT2
    m = np.where(big, m * F32(0.5), m).astype(F32)
    e = e + big.astype(np.int32)
    s = (m - F32(1.0)) / (m + F32(1.0))
    s2 = s * s
    p = _C[4]
    p = p * s2 + _C[3]
    p = p * s2 + _C[2]
    p = p * s2 + _C[1]
    p = p * s2 + _C[0]
    return e.astype(F32) * _LN2 + s * p


def synth_gumbel(w):
    w = np.asarray(w, dtype=np.uint64)
    u = ((w >> np.uint64(9)).astype(F32) + F32(0.5)) * F32(2.0 ** -23)
    t = -synth_log(u)
    return -synth_log(t)


def draft_tokens_for_rows(seed, row_ids, zd_rows, tau):
    """Drafter stand-in: one token per draft row by fp32 Gumbel-max over zD / tau."""
    rows = np.asarray(row_ids, dtype=np.int64).reshape(-1)
    zd = np.asarray(zd_rows, dtype=F32)
    V = zd.shape[-1]
    inv_tau = F32(1.0 / float(F32(tau)))
    g = synth_gumbel(words(seed, rows, SUB_DRAFT_TOKEN, V))
    score = zd * inv_tau + g
    return np.argmax(score, axis=-1).astype(np.int32)


def page_table(seed, B, N, P):
    """[B, N, P] int32 page ids: a random affine permutation of 0..B*N*P-1."""
    total = B * N * P
    rng = np.random.default_rng(int(seed) + 12345)
    A = int(rng.integers(1, max(total, 2))) | 1
    while np.gcd(A, total) != 1:
        A += 2
    Cc = int(rng.integers(0, max(total, 1)))
    i = np.arange(total, dtype=np.int64)
    return ((i * A + Cc) % total).astype(np.int32).reshape(B, N, P)


def sparse_rows(seed, rows, L, V, alpha=0.3):
    """Top-L (index, prob) rows: distinct random ids, Dirichlet(alpha) probs, sorted descending."""
    rng = np.random.default_rng(int(seed) + 777)
    idx = np.empty((rows, L), dtype=np.int32)
    for r in range(rows):
        idx[r] = rng.choice(V, size=L, replace=False)
    prob = rng.dirichlet(np.full(L, alpha), size=rows)
    order = np.argsort(-prob, axis=1, kind="stable")
    prob = np.take_along_axis(prob, order, axis=1).astype(F32)
    idx = np.take_along_axis(idx, order, axis=1)
    return idx, prob


@dataclass
class SynthConfig:
    name: str
    kind: str                 # "smc" | "verify" | "topk"
    B: int = 1
    N: int = 1
    K: int = 0
    V: int = 32000
    dtype: str = "bf16"
    sigma_z: float = 2.0
    L_head: int = 50
    sigma_d: tuple = (1.0,)   # one value, or one per third of the batch
    tau: float = 1.0
    seed: int = 0
    P: int = 0                # page-table width (pages per particle)
    topk: int = 0
    sparse_L: int = 0
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def R(self):
        return self.K + 1

    def sigma_d_of_seq(self, b):
        if len(self.sigma_d) == 1:
            return self.sigma_d[0]
        g = len(self.sigma_d)
        bounds = [round(self.B * (i + 1) / g) for i in range(g)]
        for i, hi in enumerate(bounds):
            if b < hi:
                return self.sigma_d[i]
        return self.sigma_d[-1]


CONFIGS = {
    "smc_small": SynthConfig(
        "smc_small", "smc", B=1, N=8, K=4, V=32000, dtype="f32", sigma_z=2.0, L_head=50,
        sigma_d=(0.5,), tau=1.0, seed=0, P=128,
        description="SMC-SD round, 1 sequence x 8 particles x (4+1) rows, V=32000, fp32"),
    "smc_batch": SynthConfig(
        "smc_batch", "smc", B=64, N=16, K=4, V=128256, dtype="bf16", sigma_z=2.0, L_head=50,
        sigma_d=(1.0,), tau=0.7, seed=1, P=128,
        description="SMC-SD batch, 64 x 16 x (4+1) rows, V=128256, bf16, 128-page tables"),
    "verify": SynthConfig(
        "verify", "verify", B=128, N=1, K=5, V=32000, dtype="bf16", sigma_z=2.0, L_head=50,
        sigma_d=(0.25, 1.0, 2.0), tau=1.0, seed=2,
        description="standard SD verify, 128 sequences, K=5, V=32000, bf16, draft noise by thirds"),
    "topk": SynthConfig(
        "topk", "topk", B=4096, N=1, K=0, V=152064, dtype="bf16", sigma_z=3.0, L_head=10,
        sigma_d=(0.0,), tau=0.6, seed=3, topk=8, sparse_L=10,
        description="Gumbel-top-8 over 4096 x 152064 bf16 rows; sparse 4096 x top-10 rows"),
    "smc_scale": SynthConfig(
        "smc_scale", "smc", B=256, N=32, K=8, V=128256, dtype="bf16", sigma_z=2.0, L_head=50,
        sigma_d=(1.5,), tau=1.0, seed=4, P=128,
        description="SMC-SD at scale, 256 x 32 x (8+1) rows, V=128256, bf16, 128-page tables"),
}


def row_ids_for(cfg, which, seqs=None):
    """Row ids (generator counter c1) of the target / draft tensor rows, in storage order.

    smc:    target and draft rows [B, N, K+1]: id = ((b*N)+n)*(K+1)+k.
    verify: target [B, K+1]: id = b*(K+1)+k; draft [B, K]: the paired target id.
    topk:   rows [B]: id = row.
    ``seqs`` restricts to a list of sequences b (rows of those sequences only).
    """
    seqs = np.arange(cfg.B) if seqs is None else np.asarray(seqs, dtype=np.int64)
    if cfg.kind == "smc":
        per = cfg.N * cfg.R
        return (seqs[:, None] * per + np.arange(per)[None, :]).reshape(-1)
    if cfg.kind == "verify":
        if which == "target":
            return (seqs[:, None] * cfg.R + np.arange(cfg.R)[None, :]).reshape(-1)
        return (seqs[:, None] * cfg.R + np.arange(cfg.K)[None, :]).reshape(-1)
    return seqs.copy()


def gen_config_rows(cfg, seqs=None):
    """Host-side inputs for whole sequences of a config.

    smc:    zT, zD [S, N, K+1, V], draft tokens [S, N, K]
    verify: zT [S, K+1, V], zD [S, K, V], draft tokens [S, K]
    topk:   z [S, V]
    """
    seqs = np.arange(cfg.B) if seqs is None else np.asarray(seqs, dtype=np.int64)
    S = seqs.shape[0]
    if cfg.kind == "topk":
        zt, _ = gen_rows(cfg.seed, row_ids_for(cfg, "target", seqs), cfg.V, cfg.sigma_z,
                         cfg.L_head, None, cfg.dtype)
        return dict(z=zt)
    tid = row_ids_for(cfg, "target", seqs)
    if cfg.kind == "smc":
        sd = np.array([cfg.sigma_d_of_seq(b) for b in seqs for _ in range(cfg.N * cfg.R)], dtype=F32)
        zt, zd = gen_rows(cfg.seed, tid, cfg.V, cfg.sigma_z, cfg.L_head, sd, cfg.dtype)
        zt = zt.reshape(S, cfg.N, cfg.R, cfg.V)
        zd = zd.reshape(S, cfg.N, cfg.R, cfg.V)
        did = tid.reshape(S, cfg.N, cfg.R)[:, :, :cfg.K].reshape(-1)
        x = draft_tokens_for_rows(cfg.seed, did, zd[:, :, :cfg.K].reshape(-1, cfg.V), cfg.tau)
        return dict(zT=zt, zD=zd, draft=x.reshape(S, cfg.N, cfg.K))
    # verify: draft rows exist for k < K only
    sd = np.array([cfg.sigma_d_of_seq(b) for b in seqs for _ in range(cfg.R)], dtype=F32)
    zt, zd = gen_rows(cfg.seed, tid, cfg.V, cfg.sigma_z, cfg.L_head, sd, cfg.dtype)
    zt = zt.reshape(S, cfg.R, cfg.V)
    zd = zd.reshape(S, cfg.R, cfg.V)[:, :cfg.K]
    did = row_ids_for(cfg, "draft", seqs)
    x = draft_tokens_for_rows(cfg.seed, did, zd.reshape(-1, cfg.V), cfg.tau)
    return dict(zT=zt, zD=np.ascontiguousarray(zd), draft=x.reshape(S, cfg.K))
