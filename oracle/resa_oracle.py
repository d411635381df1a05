"""Plain, slow fp64 CPU oracle of the ReSA decode hot path.

TEST INFRASTRUCTURE. Only `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline leg of `bench.py` use this module. It shares no code with the
CUDA library and imports nothing from it; the seeded input generator in
`workload/` is the only code both sides use.

Sources (all from the pages describing Rectified Sparse Attention, arXiv
2506.04108):

* "Rectified Sparse Attention" (pith.science review), section "What carries
  the argument": group block sparse attention (GBSA), in which one KV
  group's query heads share a single ranking of key blocks built from Quest's
  per-block, per-channel key minimum and maximum; after every f decode steps
  one dense causal pass recomputes the newest f tokens, overwrites their
  cached keys and values and refreshes the summaries of the blocks involved;
  the block budget n = max(n_min, ceil(M p)) (Eq. 5).
* same page, "Referee Report", major comment 1: Eq. 5 uses p as the active
  block ratio (read here as the active ratio r); Eq. 6 memory model.
* same page, minor comment 3: Eq. 2, the token mask follows its block,
  M^{ijk} = M_{ij floor(k/b)}.
* same page, "Assumptions & free parameters": b = 16, f = 32, n_min = 16,
  n_local = 1 (the newest block is always attended).
* same page, reference list: Flash-Decoding (split-KV decoding; the split is a
  schedule, the oracle computes the unsplit softmax it must equal) and Quest
  (the min/max descriptor bound).

Readings where the pages are silent:

* the Quest group score is sum over the group's heads h and channels c of
  max(q_hc * lo_c, q_hc * hi_c);
* M = ceil(len / 16) counts the partial block; ceil(M r) is computed in double
  as ceil(M r - 1e-9); n = min(M, max(n_min, ceil(M r)));
* the block holding the newest token (M - 1) is always kept and counts toward
  n; the other n - 1 are the highest scores, ties to the lower block index;
  the list is returned in ascending order;
* a decode step appends (k_new, v_new) at slot len - 1 first, then scores and
  attends, so the new token attends to itself;
* query head h reads KV head floor(h / G);
* rectify writes slots [len - f, len), recomputes every block those slots touch
  from its full contents, then runs causal dense attention in which query i
  sits at position len - f + i and sees keys 0 .. len - f + i.

Arithmetic: every value is widened to float64 before use; descriptors keep the
storage type because min/max is exact.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 16  # block size b ("Assumptions & free parameters")


# ---------------------------------------------------------------------------
# block budget, Eq. 5
# ---------------------------------------------------------------------------
def num_blocks(length: int) -> int:
    """M: number of 16-token blocks covering `length` tokens (partial counts)."""
    return (int(length) + BLOCK - 1) // BLOCK


def num_selected(M: int, r: float, n_min: int) -> int:
    """Eq. 5 with p read as the active ratio r, capped at M.

    ceil(M r) is taken in double with a 1e-9 guard so that a product that is an
    integer in exact arithmetic (e.g. 10 * 0.3) is not pushed up by binary
    rounding.
    """
    return int(min(M, max(n_min, math.ceil(M * r - 1e-9))))


# ---------------------------------------------------------------------------
# descriptors (Quest min/max per block and channel)
# ---------------------------------------------------------------------------
def build_desc(K: np.ndarray, length: int):
    """Per-block, per-channel min and max of the valid keys.

    K: [B, H, L, d]. Returns lo, hi: [B, H, M, d] (same dtype as K). Block j
    covers tokens [16 j, min(16 j + 16, length)).
    """
    M = num_blocks(length)
    B, H, _, d = K.shape
    lo = np.empty((B, H, M, d), dtype=K.dtype)
    hi = np.empty((B, H, M, d), dtype=K.dtype)
    for j in range(M):
        t0, t1 = j * BLOCK, min((j + 1) * BLOCK, length)
        seg = K[:, :, t0:t1, :]
        lo[:, :, j, :] = seg.min(axis=2)
        hi[:, :, j, :] = seg.max(axis=2)
    return lo, hi


def refresh_blocks(K: np.ndarray, lo: np.ndarray, hi: np.ndarray, length: int, j0: int):
    """Recompute descriptors of blocks j0 .. M-1 from the cache contents."""
    M = num_blocks(length)
    for j in range(j0, M):
        t0, t1 = j * BLOCK, min((j + 1) * BLOCK, length)
        seg = K[:, :, t0:t1, :]
        lo[:, :, j, :] = seg.min(axis=2)
        hi[:, :, j, :] = seg.max(axis=2)


# ---------------------------------------------------------------------------
# decode step
# ---------------------------------------------------------------------------
def group_scores(q: np.ndarray, lo: np.ndarray, hi: np.ndarray, length: int, group: int):
    """Quest upper bound pooled over each GQA group.

    q: [B, Hq, d]; lo, hi: [B, Hkv, >=M, d]. Returns s: [B, Hkv, M] float64 with
    s[..., M-1] = +inf (the local block is always kept).
    """
    M = num_blocks(length)
    B, Hq, d = q.shape
    Hkv = Hq // group
    s = np.empty((B, Hkv, M), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            qg = q[b, g * group:(g + 1) * group, :].astype(np.float64)        # [G, d]
            L = lo[b, g, :M, :].astype(np.float64)                               # [M, d]
            U = hi[b, g, :M, :].astype(np.float64)
            a = qg[:, None, :] * L[None, :, :]                                   # [G, M, d]
            c = qg[:, None, :] * U[None, :, :]
            s[b, g] = np.maximum(a, c).sum(axis=(0, 2))
    s[:, :, M - 1] = np.inf
    return s


def select_blocks(s_row: np.ndarray, n: int) -> np.ndarray:
    """Top-n blocks of one group: local block M-1, then the n-1 best others.

    Order among the others: score descending, block index ascending (ties go
    to the lower index). Returned ascending, int32.
    """
    M = s_row.shape[0]
    others = np.arange(M - 1)
    order = np.lexsort((others, -s_row[: M - 1]))   # primary: -s, secondary: index
    chosen = others[order[: n - 1]]
    return np.sort(np.concatenate([chosen, [M - 1]])).astype(np.int32)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, sel: np.ndarray, length: int,
           scale: float, group: int):
    """Softmax attention of each query head over the tokens of its group's blocks.

    q: [B, Hq, d]; K, V: [B, Hkv, L, d]; sel: [B, Hkv, n] block ids. Tokens
    t >= length are excluded (Eq. 2 applies the block mask token by token).
    Returns O [B, Hq, d] float64 and LSE [B, Hq] float64 (natural log of the
    sum of exp of the scaled logits).
    """
    B, Hq, d = q.shape
    O = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // group
            toks = np.concatenate([np.arange(j * BLOCK, min(j * BLOCK + BLOCK, length))
                                   for j in sel[b, g]])
            k = K[b, g, toks, :].astype(np.float64)
            v = V[b, g, toks, :].astype(np.float64)
            z = scale * (k @ q[b, h].astype(np.float64))
            m = z.max()
            p = np.exp(z - m)
            O[b, h] = (p @ v) / p.sum()
            lse[b, h] = m + math.log(p.sum())
    return O, lse


# ---------------------------------------------------------------------------
# prefill-side step: dense causal attention of a prompt + its descriptors
# ---------------------------------------------------------------------------
def prefill(q: np.ndarray, K: np.ndarray, V: np.ndarray, length: int, scale: float,
            group: int):
    """Causal dense attention of every prompt position, and the prompt's block
    descriptors.

    The decode loop of "Rectified Sparse Attention" (pith.science review,
    "What carries the argument") starts from a prefilled cache whose 16-token
    blocks carry Quest min/max summaries; the rectification's dense causal
    pass, applied to every position instead of the last f, is this attention.

    q: [B, len, Hq, d]; K, V: [B, Hkv, L, d] with the prompt in slots
    [0, length). Returns (O [B, len, Hq, d] float64, lo, hi) where lo/hi are
    build_desc(K, length). Query i sees keys 0 .. i.
    """
    B, L, Hq, d = q.shape
    assert L == length
    O = np.empty((B, L, Hq, d), dtype=np.float64)
    visible = np.arange(L)[None, :] <= np.arange(L)[:, None]          # [i, t]: t <= i
    for b in range(B):
        for h in range(Hq):
            g = h // group
            k = K[b, g, :L, :].astype(np.float64)
            v = V[b, g, :L, :].astype(np.float64)
            z = scale * (q[b, :, h, :].astype(np.float64) @ k.T)          # [i, t]
            z = np.where(visible, z, -np.inf)
            m = z.max(axis=1, keepdims=True)
            p = np.exp(z - m)
            O[b, :, h, :] = (p @ v) / p.sum(axis=1, keepdims=True)
    lo, hi = build_desc(K, length)
    return O, lo, hi


class State:
    """Cache + descriptors of one sequence batch, stored in the input dtype."""

    def __init__(self, K: np.ndarray, V: np.ndarray, length: int, group: int):
        self.K = np.array(K, copy=True)
        self.V = np.array(V, copy=True)
        self.length = int(length)
        self.group = int(group)
        self.lo, self.hi = build_desc(self.K, self.length)
        B, H, L, d = self.K.shape
        # capacity-sized descriptor arrays so blocks can be appended
        Mmax = L // BLOCK
        lo = np.zeros((B, H, Mmax, d), dtype=self.K.dtype)
        hi = np.zeros((B, H, Mmax, d), dtype=self.K.dtype)
        lo[:, :, : self.lo.shape[2]] = self.lo
        hi[:, :, : self.hi.shape[2]] = self.hi
        self.lo, self.hi = lo, hi

    def append(self, k_new: np.ndarray, v_new: np.ndarray):
        """Write the new token at slot `length`, then merge it into its block."""
        t = self.length
        self.K[:, :, t, :] = k_new
        self.V[:, :, t, :] = v_new
        j = t // BLOCK
        if t % BLOCK == 0:
            self.lo[:, :, j, :] = k_new
            self.hi[:, :, j, :] = k_new
        else:
            self.lo[:, :, j, :] = np.minimum(self.lo[:, :, j, :], k_new)
            self.hi[:, :, j, :] = np.maximum(self.hi[:, :, j, :], k_new)
        self.length = t + 1

    def decode(self, q, k_new, v_new, r: float, n_min: int, scale: float):
        """One sparse decode step (append, score, select, attend)."""
        if k_new is not None:
            self.append(k_new, v_new)
        M = num_blocks(self.length)
        n = num_selected(M, r, n_min)
        s = group_scores(q, self.lo, self.hi, self.length, self.group)
        B, Hkv, _ = s.shape
        sel = np.stack([np.stack([select_blocks(s[b, g], n) for g in range(Hkv)])
                        for b in range(B)])
        O, lse = attend(q, self.K, self.V, sel, self.length, scale, self.group)
        return dict(out=O, lse=lse, sel=sel, scores=s, n=n)

    def attend_with(self, q, sel, scale: float):
        """Attention over a given selection (used when the GPU's choice among
        near-tied blocks differs from the oracle's)."""
        return attend(q, self.K, self.V, np.asarray(sel), self.length, scale, self.group)

    def dense(self, q, scale: float):
        """Dense decode (every block selected): the r = 1 arm."""
        M = num_blocks(self.length)
        B, Hq, _ = q.shape
        Hkv = Hq // self.group
        sel = np.broadcast_to(np.arange(M, dtype=np.int32), (B, Hkv, M))
        return attend(q, self.K, self.V, sel, self.length, scale, self.group)

    def rectify(self, q_f, k_f, v_f, f: int, scale: float):
        """Dense rectification of the last f tokens.

        q_f: [B, f, Hq, d]; k_f, v_f: [B, f, Hkv, d]. Overwrites slots
        [len - f, len), refreshes every block those slots touch, then returns
        O_f [B, f, Hq, d] (float64) of causal dense attention, query i at
        position len - f + i seeing keys 0 .. len - f + i.
        """
        length = self.length
        t0 = length - f
        self.K[:, :, t0:length, :] = np.transpose(k_f, (0, 2, 1, 3))
        self.V[:, :, t0:length, :] = np.transpose(v_f, (0, 2, 1, 3))
        refresh_blocks(self.K, self.lo, self.hi, length, t0 // BLOCK)
        B, _, Hq, d = q_f.shape
        G = self.group
        O = np.empty((B, f, Hq, d), dtype=np.float64)
        for b in range(B):
            for g in range(Hq // G):
                k = self.K[b, g, :length, :].astype(np.float64)      # [len, d]
                v = self.V[b, g, :length, :].astype(np.float64)
                for hh in range(G):
                    h = g * G + hh
                    qh = q_f[b, :, h, :].astype(np.float64)           # [f, d]
                    z = scale * (qh @ k.T)                            # [f, len]
                    pos = t0 + np.arange(f)
                    visible = np.arange(length)[None, :] <= pos[:, None]
                    z = np.where(visible, z, -np.inf)
                    m = z.max(axis=1, keepdims=True)
                    p = np.exp(z - m)
                    O[b, :, h, :] = (p @ v) / p.sum(axis=1, keepdims=True)
        return O
