"""Property pins of the oracle attention on random shapes (hypothesis):
outputs are convex combinations of value rows (inside their per-channel
range), joint key/value permutations leave outputs unchanged, query
permutations permute them, and a key-length mask equals dropping the
masked rows.  A transposed operand, a wrong softmax axis or a mask applied
to the wrong side breaks at least one of them."""

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import attention as oattn


@st.composite
def problems(draw):
    lq = draw(st.integers(1, 12))
    lk = draw(st.integers(1, 12))
    d = draw(st.sampled_from([4, 8, 16]))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    scale = draw(st.floats(0.05, 3.0))
    r = np.random.default_rng(seed)
    return (r.standard_normal((lq, d)), r.standard_normal((lk, d)),
            r.standard_normal((lk, d)) * 3, scale, r)


@settings(max_examples=60, deadline=None)
@given(problems())
def test_output_in_value_hull(p):
    q, k, v, scale, _ = p
    o = oattn.attend(q, k, v, scale)
    lo, hi = v.min(0), v.max(0)
    assert np.all(o >= lo - 1e-12) and np.all(o <= hi + 1e-12)


@settings(max_examples=60, deadline=None)
@given(problems())
def test_permutation_equivariance(p):
    q, k, v, scale, r = p
    o = oattn.attend(q, k, v, scale)
    pk = r.permutation(k.shape[0])
    assert np.allclose(oattn.attend(q, k[pk], v[pk], scale), o, atol=1e-12)
    pq = r.permutation(q.shape[0])
    assert np.allclose(oattn.attend(q[pq], k, v, scale), o[pq], atol=1e-12)


@settings(max_examples=60, deadline=None)
@given(problems())
def test_key_length_equals_dropping_rows(p):
    q, k, v, scale, r = p
    n = int(r.integers(1, k.shape[0] + 1))
    masked = oattn.attend(q, k, v, scale, kv_len=n)
    assert np.allclose(masked, oattn.attend(q, k[:n], v[:n], scale),
                       atol=1e-12)
