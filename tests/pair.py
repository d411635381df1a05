"""GPU path and CPU oracle driven side by side on the same seeded inputs.

Both sides receive identical values from the workload generator; nothing the
GPU computes is fed back into the oracle, except that a near-tied selection
(gap rule below) is re-evaluated by the oracle on the GPU's block list.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from workload import Spec, decode_inputs, make_cache, rectify_inputs

# tolerances: bf16 K/V rel-L2 <= 5e-3 and max-abs <= 2e-2; fp32 both <= 1e-5
TOL = {"bf16": (5e-3, 2e-2), "f32": (1e-5, 1e-5)}
GAP = 1e-4   # relative gap between the n-th and (n+1)-th oracle score


def tdt(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    # values are exactly representable in `dtype`; the conversion is exact
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(tdt(dtype))


def close(got, ref, dtype: str, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rel_tol, abs_tol = TOL[dtype]
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(diff).max() if diff.size else 0.0
    assert rel <= rel_tol and mx <= abs_tol, f"{what}: rel-L2 {rel:.3e} max-abs {mx:.3e}"
    return rel, mx


# (step, KV group) decisions seen by check_selection: "exact" ones were
# asserted equal to the oracle's set, "near_tie" ones passed the band checks
SELECTION_STATS = {"exact": 0, "near_tie": 0}


def fp32_score_error(q: np.ndarray, lo: np.ndarray, hi: np.ndarray, M: int) -> np.ndarray:
    """Bound on |fp32 score - exact score| for every block of every group.

    The kernel folds the group into N_c = sum_h min(q_hc, 0) and
    P_c = sum_h max(q_hc, 0) (G fp32 additions) and sums the 2d products
    N_c lo_c and P_c hi_c in some fp32 order; whatever the order, the error
    of such a sum is at most gamma_k times the sum of the products' magnitudes
    (gamma_k = k u / (1 - k u), u = 2^-24, k >= number of rounded operations
    on any path), and that sum is at most sum_c (sum_h |q_hc|) max(|lo_c|, |hi_c|).
    q: [B, Hq, d]; lo, hi: [B, Hkv, >= M, d]. Returns [B, Hkv, M]."""
    B, Hq, d = q.shape
    H = lo.shape[1]
    G = Hq // H
    k = 2 * d + G + 2
    u = 2.0 ** -24
    gamma = k * u / (1.0 - k * u)
    qa = np.abs(np.asarray(q, np.float64)).reshape(B, H, G, d).sum(axis=2)       # [B, H, d]
    mx = np.maximum(np.abs(np.asarray(lo[:, :, :M], np.float64)),
                    np.abs(np.asarray(hi[:, :, :M], np.float64)))                # [B, H, M, d]
    return gamma * np.einsum("bhmd,bhd->bhm", mx, qa)


def check_selection(gpu_sel: np.ndarray, scores: np.ndarray, n: int,
                    err: np.ndarray | None = None) -> bool:
    """Selection parity on one (batch, KV group).

    s_(n) and s_(n+1) are the oracle's (n-1)-th and n-th best scores among the
    non-local blocks (the local block takes one of the n places). Where their
    relative gap exceeds GAP the GPU set must equal the oracle's bit-exactly.
    Otherwise (a near tie, where fp32 and fp64 scores may order blocks
    differently) with the band B = [s_(n+1) - d, s_(n) + d], d = GAP |s_(n)|:
      * every non-local block scoring above B is selected;
      * every other selected block scores inside B (so the list holds exactly
        n - 1 - #above of them);
      * no unselected block beats a selected one by more than d.
    With `err` (a bound on each block's fp32 score error, fp32_score_error),
    a near tie whose oracle set is separated from the rest by more than the
    error bounds (min over kept of s - err > max over the others of s + err)
    cannot be reordered by fp32 rounding, so it must be exact as well.
    Returns True for an exact decision, False for a near tie."""
    M = scores.shape[0]
    sel = [int(x) for x in gpu_sel]
    assert len(sel) == n, (len(sel), n)
    assert sel == sorted(set(sel)), "selection must be ascending and unique"
    assert sel[-1] == M - 1 and sel[0] >= 0, "local block must be kept"
    oracle_sel = [int(x) for x in orc.select_blocks(scores, n)]
    if n == 1 or n >= M:
        assert sel == oracle_sel
        SELECTION_STATS["exact"] += 1
        return True
    others = np.asarray(scores[: M - 1], dtype=np.float64)
    order = np.lexsort((np.arange(M - 1), -others))
    s_n, s_next = others[order[n - 2]], others[order[n - 1]]
    d = GAP * max(abs(s_n), 1e-30)
    if (s_n - s_next) > d:
        assert sel == oracle_sel, "selection differs although the score gap is clear"
        SELECTION_STATS["exact"] += 1
        return True
    if err is not None:
        e = np.asarray(err[: M - 1], dtype=np.float64)
        kept, rest_o = order[: n - 1], order[n - 1:]
        if (others[kept] - e[kept]).min() > (others[rest_o] + e[rest_o]).max():
            assert sel == oracle_sel, "selection differs although fp32 error cannot reorder it"
            SELECTION_STATS["exact"] += 1
            return True
    chosen = np.asarray(sel[:-1], dtype=np.int64)
    picked = np.zeros(M - 1, dtype=bool)
    picked[chosen] = True
    above = others > s_n + d
    assert np.all(picked[above]), "a block scoring above the near-tie band was dropped"
    rest = others[picked & ~above]
    assert np.all(rest >= s_next - d), "selected a block below the near-tie band"
    assert rest.size == (n - 1) - int(above.sum())
    if np.any(~picked):
        assert others[picked].min() >= others[~picked].max() - d, \
            "an unselected block beats a selected one by more than the band"
    SELECTION_STATS["near_tie"] += 1
    return False


class Pair:
    """GPU state (torch tensors) + oracle state for one workload."""

    def __init__(self, spec: Spec, n_min: int | None = None, r: float | None = None,
                 cache=None, rows=None):
        """rows: batch rows the oracle mirrors (all by default); batch rows
        are independent, so a subset keeps large cases cheap on the CPU."""
        self.spec = spec
        import block_sparse_attention_quest_b200 as resa
        self.resa = resa
        self.r = spec.r if r is None else r
        self.n_min = spec.n_min if n_min is None else n_min
        K, V = make_cache(spec) if cache is None else cache
        self.rows = list(range(spec.batch)) if rows is None else list(rows)
        self.st = orc.State(K[self.rows], V[self.rows], spec.len0, spec.group)
        self.k = to_dev(K, spec.dtype)
        self.v = to_dev(V, spec.dtype)
        self.desc = torch.zeros(spec.batch, spec.n_kv_heads, spec.max_blocks, 2, spec.head_dim,
                                dtype=tdt(spec.dtype), device="cuda")
        self.length = spec.len0
        resa.build_desc(self.k, self.length, self.desc, spec.n_q_heads)
        self.dims = resa.dims_for(self.k, spec.n_q_heads)
        self.ws = resa.alloc_workspace(self.dims, spec.max_len, max(spec.f, 64))
        self.rect_calls = 0

    def desc_matches(self):
        M = orc.num_blocks(self.length)
        d = self.desc[self.rows, :, :M].float().cpu().numpy()
        return (np.array_equal(d[:, :, :, 0], self.st.lo[:, :, :M]) and
                np.array_equal(d[:, :, :, 1], self.st.hi[:, :, :M]))

    def decode(self, step: int, check: bool = True, dense: bool = False, scale: float = 1.0):
        spec = self.spec
        q, kn, vn = decode_inputs(spec, step)
        self.length += 1
        out = torch.empty(spec.batch, spec.n_q_heads, spec.head_dim, dtype=tdt(spec.dtype),
                          device="cuda")
        lse = torch.empty(spec.batch, spec.n_q_heads, dtype=torch.float32, device="cuda")
        if dense:
            self.resa.decode_dense(to_dev(q, spec.dtype), to_dev(kn, spec.dtype),
                                   to_dev(vn, spec.dtype), self.k, self.v, self.desc, self.length,
                                   scale, out, self.ws, lse=lse)
            sel = None
        else:
            n = self.resa.num_selected(self.length, self.r, self.n_min)
            sel = torch.empty(spec.batch, spec.n_kv_heads, n, dtype=torch.int32, device="cuda")
            self.resa.decode_sparse(to_dev(q, spec.dtype), to_dev(kn, spec.dtype),
                                    to_dev(vn, spec.dtype), self.k, self.v, self.desc, self.length,
                                    self.r, self.n_min, scale, out, self.ws, lse=lse, sel=sel)
        assert self.resa.workspace_status(self.ws) == self.resa.RESA_OK
        R = self.rows
        q, kn, vn = q[R], kn[R], vn[R]
        out, lse = out[R], lse[R]
        if dense:
            self.st.append(kn, vn)
            O, L = self.st.dense(q, scale)
            res = dict(out=O, lse=L, exact=True)
        else:
            res = self.st.decode(q, kn, vn, self.r, self.n_min, scale)
            gsel = sel[R].cpu().numpy()
            M = res["scores"].shape[-1]
            err = fp32_score_error(q, self.st.lo, self.st.hi, M)
            exact = True
            for b in range(len(R)):
                for g in range(spec.n_kv_heads):
                    exact &= check_selection(gsel[b, g], res["scores"][b, g], res["n"],
                                             err[b, g])
            if not exact:   # near-tie somewhere: compare on the GPU's selection
                O, L = self.st.attend_with(q, gsel, scale)
                res = dict(res, out=O, lse=L)
            res["exact"] = exact
            res["gpu_sel"] = gsel
        if check:
            close(out.float().cpu().numpy(), res["out"], spec.dtype, f"decode step {step} out")
            close(lse.cpu().numpy(), res["lse"], "f32" if spec.dtype == "f32" else "bf16",
                  f"decode step {step} lse")
        return res

    def rectify(self, f: int | None = None, check: bool = True, scale: float = 1.0):
        spec = self.spec
        f = spec.f if f is None else f
        q_f, k_f, v_f = rectify_inputs(spec, self.rect_calls, self.length, f)
        self.rect_calls += 1
        out = torch.empty(spec.batch, f, spec.n_q_heads, spec.head_dim, dtype=tdt(spec.dtype),
                          device="cuda")
        self.resa.rectify(to_dev(q_f, spec.dtype), to_dev(k_f, spec.dtype), to_dev(v_f, spec.dtype),
                          self.k, self.v, self.desc, self.length, f, scale, out, self.ws)
        assert self.resa.workspace_status(self.ws) == self.resa.RESA_OK
        R = self.rows
        ref = self.st.rectify(q_f[R], k_f[R], v_f[R], f, scale)
        if not check:
            return None
        close(out[R].float().cpu().numpy(), ref, spec.dtype, f"rectify f={f} at len {self.length}")
        return ref
