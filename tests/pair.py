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


def check_selection(gpu_sel: np.ndarray, scores: np.ndarray, n: int):
    """Gap rule on one (b, g). Returns True when the GPU set must equal the
    oracle's (and does); False when near-tied (the GPU choice is then only
    checked for validity)."""
    M = scores.shape[0]
    sel = [int(x) for x in gpu_sel]
    assert len(sel) == n, (len(sel), n)
    assert sel == sorted(set(sel)), "selection must be ascending and unique"
    assert sel[-1] == M - 1 and sel[0] >= 0, "local block must be kept"
    oracle_sel = [int(x) for x in orc.select_blocks(scores, n)]
    if n == 1 or n >= M:
        assert sel == oracle_sel
        return True
    others = scores[: M - 1]
    order = np.lexsort((np.arange(M - 1), -others))
    s_n, s_next = others[order[n - 2]], others[order[n - 1]]
    scale = max(abs(s_n), 1e-30)
    if (s_n - s_next) / scale > GAP:
        assert sel == oracle_sel, "selection differs although the score gap is clear"
        return True
    thr = s_next - GAP * scale
    assert all(others[j] >= thr for j in sel[:-1]), "selected a block below the near-tie band"
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
            exact = True
            for b in range(len(R)):
                for g in range(spec.n_kv_heads):
                    exact &= check_selection(gsel[b, g], res["scores"][b, g], res["n"])
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
