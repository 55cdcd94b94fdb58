"""The seeded input generator: distributions, determinism, bf16 rounding."""
import numpy as np
import torch

import inputgen as IG
from inputgen.workloads import Workload, NORMAL, UNIFORM, ZERO, ONES, ALL, rope_split

W0 = Workload("gen", B=1, H=8, D=128, fh=16, fw=32, C=2, S=1, W=2, n_chunks=1, dtype="f32")


def test_normal_moments_and_support():
    x = IG.fill_host(W0, 0, 0, IG.Q).ravel().astype(np.float64)  # 1M values
    assert abs(x.mean()) < 5e-3
    assert abs(x.var() - 1.0) < 5e-3
    assert np.abs(x).max() <= 6.0
    # Irwin-Hall(12) kurtosis is 3 - 1.2/12 = 2.9
    k = ((x - x.mean()) ** 4).mean() / x.var() ** 2
    assert abs(k - 2.9) < 0.03


def test_uniform_moments_and_support():
    w = W0.with_(dist=(UNIFORM, UNIFORM, UNIFORM))
    x = IG.fill_host(w, 0, 0, IG.V).ravel().astype(np.float64)
    assert x.min() > -1.0 and x.max() < 1.0
    assert abs(x.mean()) < 3e-3
    assert abs(x.var() - 1.0 / 3.0) < 3e-3


def test_constants():
    w = W0.with_(dist=(ZERO, ONES, NORMAL))
    assert not IG.fill_host(w, 0, 0, IG.Q).any()
    assert (IG.fill_host(w, 0, 0, IG.K) == 1.0).all()


def test_bf16_rounding_matches_torch_cast():
    x32 = IG.fill_host(W0, 3, 5, IG.K)
    bits = IG.fill_host(W0.with_(dtype="bf16"), 3, 5, IG.K)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)


def test_determinism_offsets_and_independence():
    a = IG.fill_host(W0, 1, 7, IG.Q)
    b = IG.fill_host(W0, 1, 7, IG.Q)
    np.testing.assert_array_equal(a, b)
    part = IG.fill_host(W0, 1, 7, IG.Q, tok0=100, n_tok=37)
    np.testing.assert_array_equal(part, a[100:137])
    for other in (IG.fill_host(W0, 2, 7, IG.Q), IG.fill_host(W0, 1, 8, IG.Q),
                  IG.fill_host(W0, 1, 7, IG.K), IG.fill_host(W0.with_(seed=1), 1, 7, IG.Q)):
        assert np.mean(other == a) < 0.01


def test_outlier_rows():
    w = W0.with_(outlier_frac=0.01, outlier_scale=20.0)
    plain = IG.fill_host(W0, 0, 0, IG.K).reshape(-1, W0.D)
    out = IG.fill_host(w, 0, 0, IG.K).reshape(-1, W0.D)
    ratio_rows = np.all(out == plain * 20.0, axis=1)
    same_rows = np.all(out == plain, axis=1)
    assert np.all(ratio_rows | same_rows)
    frac = ratio_rows.mean()
    assert 0.008 < frac < 0.012, frac
    # only K carries outliers
    np.testing.assert_array_equal(IG.fill_host(w, 0, 0, IG.Q), IG.fill_host(W0, 0, 0, IG.Q))


def test_workload_table():
    names = [w.name for w in ALL]
    assert len(set(names)) == 5
    assert rope_split(128) == (44, 42, 42) and rope_split(64) == (24, 20, 20)
    for w in ALL:
        assert sum(w.dims) == w.D and all(d % 2 == 0 for d in w.dims)
        assert len(w.start_steps) == w.B
    long = [w for w in ALL if w.B == 8][0]
    assert long.n_steps == 42 + 10000
    assert long.local_chunks(5) == [5, 2, -1, -1, -1, -1, -1, -1]
