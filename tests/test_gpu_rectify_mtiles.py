"""Dense rectification with more than 128 query rows per KV head (f * G >
128): several 128-row m-tiles per KV head, the CTAs of one split's m-tiles
launched side by side so that they stream the same key tiles together,
against the oracle.

"Rectified Sparse Attention" (pith.science review), section "What carries the
argument": the rectification re-encodes the newest f tokens by dense causal
attention over the whole cache."""
import pytest

from pair import Pair
from workload import Spec

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("hq,hkv,d,length,f", [
    (16, 4, 64, 700, 64),     # two m-tiles, head_dim 64
    (16, 2, 128, 1500, 33),   # group 8: 264 rows, three m-tiles (the last one mostly padding)
    (8, 2, 128, 2000, 100),   # four m-tiles
    (4, 2, 64, 300, 100),     # group 2: 200 rows
    (8, 2, 128, 129, 64),     # one full key tile and one key
])
def test_multi_mtile_shapes(hq, hkv, d, length, f):
    spec = Spec(batch=2, n_q_heads=hq, n_kv_heads=hkv, head_dim=d, len0=length, steps=0,
                dtype="bf16", f=f, max_len=((length + 15) // 16) * 16 + 32)
    p = Pair(spec)
    p.rectify(f)
    assert p.desc_matches()


def test_multi_mtile_stale_slots_do_not_leak():
    """Slots at or past len hold NaN bit patterns; the rows of the last key
    tile past the end of the cache must not reach an output."""
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=1000, steps=0,
                dtype="bf16", f=64, max_len=1056)
    p = Pair(spec)
    p.k[:, :, spec.len0:] = float("nan")
    p.v[:, :, spec.len0:] = float("nan")
    p.rectify(64)


def test_multi_mtile_one_split_per_unit():
    """Enough (batch row, KV head, m-tile) units to fill the GPU: no key
    splits, the output written by the kernel itself."""
    spec = Spec(batch=38, n_q_heads=16, n_kv_heads=4, head_dim=128, len0=300, steps=0,
                dtype="bf16", f=64, max_len=352)
    p = Pair(spec)
    p.rectify(64)
    assert p.desc_matches()
