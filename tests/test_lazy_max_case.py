"""CPU checks of the inputs the lazy-max GPU test builds (tests/test_gpu_decode_exact.py):
they are bf16 values, each head's special row lands on opposite sides of the
rescale threshold in the two roundings a CTA pair applies, and a merge that
used one CTA's softmax statistics for both latent halves would miss the
tolerance by far, so the GPU test can tell the two merges apart."""
import math

import numpy as np
import pytest

from head_latent_attention_decode_b200 import workloads as wl

from test_gpu_decode_exact import _threshold_combos, lazy_max_case


def _f16(x):
    return np.float16(x).astype(np.float64)


@pytest.mark.parametrize("name,special,tile", [("v2lite_bf16", 130, 128), ("v3_bf16", 70, 64)])
def test_lazy_max_case_straddles_and_separates_the_merges(name, special, tile):
    s = wl.WORKLOADS[name].shape
    n, L = 4, 2048
    q_abs, q_pe, cache, table, lens = lazy_max_case(s, n, L, special)
    assert special // tile == 1 and special < 2 * tile   # second tile of the first split
    c = float(np.float32(1.0 / math.sqrt(s.qk_nope + s.qk_rope)) * np.float32(1.4426950408889634))
    bs = s.block_size
    worst_ratio = 0.0
    for h in range(s.n_heads):
        b = h % n
        rows = np.array([table[b, j // bs] * bs + j % bs for j in range(L)])
        a0, a1 = q_abs[b, h, h], q_abs[b, h, 256 + h]
        S0 = a0 * cache[rows, h].astype(np.float64)       # first CTA's partial (exact)
        S1 = a1 * cache[rows, 256 + h].astype(np.float64)  # second CTA's partial (exact)
        views = (S0 + _f16(S1), _f16(S0) + S1)             # own fp32 + peer f16, per CTA
        assert np.all(views[0][:special] == 0) and np.all(views[1][:special] == 0)
        above = [v[special] * c > 8.0 for v in views]
        assert above[0] != above[1], h                     # the CTAs disagree on the rescale
        # each CTA's reference max after the first split's tiles, and its sum
        m = [v[special] * c if up else 0.0 for v, up in zip(views, above)]
        l = [np.sum(2.0 ** (v * c - mr)) for v, mr in zip(views, m)]
        # one split holding everything: the half normalised with the other CTA's
        # statistics is off by 2^(m_1 - m_0) against its own
        ratio = (2.0 ** (m[0] - m[1])) * (l[1] / l[0])
        worst_ratio = max(worst_ratio, abs(math.log2(ratio)))
    assert worst_ratio > 7.0   # a factor of more than 2^7 on half of o_lat
