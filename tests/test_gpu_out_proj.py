"""GPU parity of the grouped output projection ("DeepSeek-V4: million-token
context" section 4.4) against the fp64 oracle.  The library keeps the
intermediate z in bf16 and writes y in bf16 (fp32 accumulation), so each
element of y may differ from the exact one by at most
  2^-9 sum_k |z_k| |W2_jk|  (z rounded to bf16)
+ 2^-9 |y_j|                 (y rounded to bf16)
+ fp32 accumulation, bounded by 2^-16 of the absolute sums of both products;
the test checks that bound element by element."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_11_b200 as csa
import csa_inputs as G
import oracle as O
from _util import host

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _weights(Gr, dg, kin, d, seed):
    w1 = G.normal((Gr, dg, kin), seed, 60, std=kin ** -0.5, dtype=torch.bfloat16)
    w2 = G.normal((d, Gr * dg), seed, 61, std=(Gr * dg) ** -0.5, dtype=torch.bfloat16)
    return w1, w2


def _check(got, o, w1, w2):
    o64, W1, W2 = O.f64(o), O.f64(w1), O.f64(w2)
    n, nh, c = o64.shape
    Gr = W1.shape[0]
    hpg = nh // Gr
    z = np.concatenate([o64[:, g * hpg:(g + 1) * hpg].reshape(n, -1) @ W1[g].T
                        for g in range(Gr)], axis=1)
    zabs = np.concatenate([np.abs(o64[:, g * hpg:(g + 1) * hpg].reshape(n, -1)) @ np.abs(W1[g]).T
                           for g in range(Gr)], axis=1)
    ref = O.grouped_output_projection(o64, W1, W2)
    assert np.allclose(ref, z @ W2.T)
    bound = 2.0 ** -9 * (np.abs(z) @ np.abs(W2).T) + 2.0 ** -9 * np.abs(ref) + \
        2.0 ** -16 * (zabs @ np.abs(W2).T + np.abs(z) @ np.abs(W2).T) + 1e-6
    err = np.abs(O.f64(got) - ref)
    assert np.all(np.isfinite(O.f64(got)))
    assert np.all(err <= bound), (float(err.max()), float((err / bound).max()))


@pytest.mark.parametrize("rows,nh,c,Gr,dg,d", [
    (300, 64, 512, 8, 256, 512),     # ragged row count (300 = 2 x 128 + 44)
    (129, 16, 128, 4, 256, 256),
    (64, 8, 64, 1, 256, 768),        # one group: a plain two-step projection
])
def test_grouped_out_proj_matches_oracle(rows, nh, c, Gr, dg, d):
    o = G.normal((rows, nh, c), 62, 1, dtype=torch.bfloat16)
    w1, w2 = _weights(Gr, dg, nh // Gr * c, d, 62)
    y = host(csa.csa_grouped_out_proj(o.to(DEV), w1.to(DEV), w2.to(DEV)))
    csa.csa_check()
    _check(y, o, w1, w2)


def test_grouped_out_proj_flash_shape_sampled_rows():
    """V4-Flash: 64 heads x 512 in 8 groups, d_g = 1024, d = 4096, on 4096
    rows; sampled rows against the oracle."""
    rows, nh, c, Gr, dg, d = 4096, 64, 512, 8, 1024, 4096
    o = G.normal((rows, nh, c), 63, 1, dtype=torch.bfloat16)
    w1, w2 = _weights(Gr, dg, nh // Gr * c, d, 63)
    y = host(csa.csa_grouped_out_proj(o.to(DEV), w1.to(DEV), w2.to(DEV)))
    csa.csa_check()
    pick = [0, 1, 127, 128, 2047, 2048, 4000, 4095]
    _check(y[pick], o[pick], w1, w2)
