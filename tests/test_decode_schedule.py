"""The streaming decode kernel's order of work, replayed in numpy on the host:
a KV head's cache rows split into chunks of whole 64-row tiles, each tile's
keys dealt to key slices (key c of a tile to slice c mod SL), every slice
keeping its own running maximum M and sum l in base 2 (per tile: the slice's
maximum, the rescale factor 2^(M_old - M) and p = 2^(x - M), with M taken as 0
while the slice has seen no key), then the slices rescaled to the largest slice
maximum and added in slice order, then the chunks merged the same way.  That
reordering must give the softmax-weighted sum of the values, exactly up to
rounding, whatever the chunk and slice sizes; checked against the oracle's
decode attention, with chunks so short that most slices never see a key."""
import math

import numpy as np
import pytest

from oracle import tokengate_oracle as O

R = 64  # cache rows per tile


def _replay(x2, v, chunk, slices):
    """x2: [L] base-2 logits of one head; v: [L][D] values -> output [D]."""
    length = x2.shape[0]
    parts = []
    for c0 in range(0, length, chunk):
        nk = min(chunk, length - c0)
        m = np.full(slices, -np.inf)
        l = np.zeros(slices)
        acc = np.zeros((slices, v.shape[1]))
        for t0 in range(0, nk, R):
            keys = np.arange(t0, t0 + R)
            xt = np.where(keys < nk, x2[c0 + np.minimum(keys, nk - 1)], -np.inf)
            for s in range(slices):
                mine = np.arange(s, R, slices)
                m_new = max(m[s], xt[mine].max())
                m_use = 0.0 if m_new == -np.inf else m_new
                alpha = 2.0 ** (m[s] - m_use)
                m[s] = m_new
                l[s] *= alpha
                acc[s] *= alpha
                for c in mine:
                    p = 2.0 ** (xt[c] - m_use)
                    l[s] += p
                    if t0 + c < nk:
                        acc[s] += p * v[c0 + t0 + c]
        mx = m.max()
        w = 2.0 ** (m - mx)
        parts.append((mx, (w * l).sum(), (w[:, None] * acc).sum(0)))
    mx = max(p[0] for p in parts)
    wts = [2.0 ** (p[0] - mx) for p in parts]
    total = sum(w * p[1] for w, p in zip(wts, parts))
    return sum(w * p[2] for w, p in zip(wts, parts)) / total


@pytest.mark.parametrize("length,chunk,slices", [(1, 64, 8), (63, 64, 8), (200, 128, 8), (517, 192, 16),
                                                 (700, 64, 5), (1333, 448, 2), (2129, 128, 8)])
def test_streaming_decode_order_equals_the_oracle(length, chunk, slices):
    rng = np.random.default_rng(length * 7 + slices)
    hq, hkv, dh = 2, 1, 16
    q = rng.standard_normal((hq, dh))
    k = rng.standard_normal((length, hkv, dh))
    v = rng.standard_normal((length, hkv, dh))
    bias = rng.standard_normal(length)
    gain = rng.uniform(0.5, 2.0, hq)
    temp = rng.uniform(0.8, 1.2, hq)
    ratio, sm_scale = 0.9, 1.0 / math.sqrt(dh)
    want = O.gated_decode_attention(q, k, v, bias, gain, temp, ratio, sm_scale)
    log2e = 1.0 / math.log(2.0)
    for h in range(hq):
        x2 = (temp[h] * ratio * sm_scale * log2e) * (k[:, 0, :] @ q[h]) + gain[h] * log2e * bias
        got = _replay(x2, v[:, 0, :], chunk, slices)
        np.testing.assert_allclose(got, want[h], rtol=1e-12, atol=1e-12)
