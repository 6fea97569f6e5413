"""The GLU-MLP mapping of the hybrid format (SpenseGPT): the oracle pinned by
the cases that reduce to plain computations -- no pruning (dense MLP), no
dense share (every projection plain 2:4), the permutation being absorbed
(packed weights in permuted order reproduce the original-order result), the
dense set being the top of the summed score, and SiLU's closed forms."""
import numpy as np
import pytest

import oracle
from semi_structured_sparse_nm_b200 import inputs


def _mlp(rng_seed, I=1024, d=256, T=6):
    wu = inputs.normal_bf16((I, d), 0.02, rng_seed)
    wg = inputs.normal_bf16((I, d), 0.02, rng_seed + 1)
    wd = inputs.normal_bf16((d, I), 0.02, rng_seed + 2)
    x = inputs.normal_bf16((T, d), 1.0, rng_seed + 3)
    return x, wu, wg, wd


def _dense_mlp(x, wu, wg, wd, ku=None, kg=None, kd=None):
    f = inputs.bf16_to_f64
    U = f(wu) * (1 if ku is None else ku)
    G = f(wg) * (1 if kg is None else kg)
    Dn = f(wd) * (1 if kd is None else kd)
    g = f(x) @ G.T
    h = (g / (1.0 + np.exp(-g))) * (f(x) @ U.T)
    return h @ Dn.T


def test_silu_closed_forms():
    z = np.array([0.0, 40.0, -40.0, 1.0, -2.5])
    s = oracle.silu_f64(z)
    assert s[0] == 0.0 and abs(s[1] - 40.0) < 1e-12 and abs(s[2]) < 1e-15
    assert np.allclose(s[3:], z[3:] / (1.0 + np.exp(-z[3:])), rtol=0, atol=1e-15)


def test_all_dense_is_the_dense_mlp():
    x, wu, wg, wd = _mlp(10)
    y = oracle.spense_mlp(x, wu, wg, wd, 1.0)
    assert np.allclose(y, _dense_mlp(x, wu, wg, wd), rtol=1e-12, atol=1e-15)


def test_no_dense_share_is_plain_two_four_everywhere():
    x, wu, wg, wd = _mlp(20)
    p = oracle.spense_mlp_weights(wu, wg, wd, 0.0)
    assert p["D"] == 0 and np.array_equal(p["perm"], np.arange(wu.shape[0]))
    ku, kg, kd = oracle.prune(wu, 2, 4), oracle.prune(wg, 2, 4), oracle.prune(wd, 2, 4)
    assert np.array_equal(p["keep_up"], ku) and np.array_equal(p["keep_gate"], kg)
    assert np.array_equal(p["keep_down"], kd)
    assert np.allclose(oracle.spense_mlp(x, wu, wg, wd, 0.0), _dense_mlp(x, wu, wg, wd, ku, kg, kd),
                       rtol=1e-12, atol=1e-15)


def test_dense_set_is_the_top_of_the_summed_score():
    x, wu, wg, wd = _mlp(30)
    p = oracle.spense_mlp_weights(wu, wg, wd, 0.25)
    f = inputs.bf16_to_f64
    score = (f(wu) ** 2).sum(1) + (f(wg) ** 2).sum(1) + (f(wd) ** 2).sum(0)
    assert np.allclose(p["score"], score, rtol=1e-13)
    order = np.argsort(-p["score"], kind="stable")
    assert set(order[:p["D"]]) == set(np.flatnonzero(p["is_dense"]))
    assert p["D"] == 256 and np.array_equal(p["perm"][p["Is"]:], np.sort(order[:p["D"]]))


@pytest.mark.parametrize("frac", [0.25, 0.5])
def test_permuted_packing_reproduces_the_original_order(frac):
    """The packed weights, used in the permuted order (output-split up/gate,
    input-split down), give the same MLP as the original order: the
    permutation of the intermediate indices is absorbed."""
    x, wu, wg, wd = _mlp(40)
    p = oracle.spense_mlp_weights(wu, wg, wd, frac)
    I, d = wu.shape
    Is, D = p["Is"], p["D"]
    ug_s = oracle.decompress(p["ug_vals"], oracle.compress(
        np.concatenate([wu[p["perm"][:Is]], wg[p["perm"][:Is]]]),
        np.concatenate([p["keep_up"][p["perm"][:Is]], p["keep_gate"][p["perm"][:Is]]]), 4)[1], d, 4)
    f = inputs.bf16_to_f64
    ug = np.concatenate([f(ug_s), f(p["ug_dense"])])            # rows [up_s; gate_s; up_d; gate_d]
    up_rows = np.concatenate([ug[:Is], ug[2 * Is:2 * Is + D]])
    gate_rows = np.concatenate([ug[Is:2 * Is], ug[2 * Is + D:]])
    g = f(x) @ gate_rows.T
    h = (g / (1.0 + np.exp(-g))) * (f(x) @ up_rows.T)           # intermediate values in permuted order
    kd_s = oracle.compress(np.ascontiguousarray(oracle.gather_cols(wd, p["perm"])[:, :Is]),
                           p["keep_down"][:, p["perm"][:Is]], 4)[1]
    down = np.concatenate([f(oracle.decompress(p["down_vals"], kd_s, Is, 4)), f(p["down_dense"])], axis=1)
    y_perm = h @ down.T
    assert np.allclose(y_perm, oracle.spense_mlp(x, wu, wg, wd, frac), rtol=1e-10, atol=1e-14)


def test_rownorm_exact_on_integers_and_the_transpose_of_colnorm():
    rng = np.random.default_rng(21)
    wi = rng.integers(-9, 10, size=(48, 200))
    w = inputs.bf16_from_f64(wi.astype(np.float64))
    exact = np.array([sum(int(v) * int(v) for v in row) for row in wi], dtype=np.float64)
    assert np.array_equal(oracle.rownorm_f64(w), exact)
    g = inputs.normal_bf16((64, 96), 0.02, seed=22)
    assert np.array_equal(oracle.rownorm_f64(g), oracle.colnorm_f64(np.ascontiguousarray(g.T)))


@pytest.mark.parametrize("I", [256, 1024, 14336])
def test_dense_count_invariants(I):
    """Whole blocks of 256 intermediate indices, never above the share f * I
    and within one block of it; nothing at f <= 0, everything at f >= 1."""
    for f in (0.05, 0.25, 0.3, 0.5, 0.99):
        D = oracle.spense_dense_count(I, f)
        assert D % 256 == 0 and D <= f * I < D + 256, (I, f, D)
    assert oracle.spense_dense_count(I, 0.0) == 0 and oracle.spense_dense_count(I, -1.0) == 0
    assert oracle.spense_dense_count(I, 1.0) == I and oracle.spense_dense_count(I, 2.0) == I
    if I == 14336:
        assert oracle.spense_dense_count(I, 0.25) == 3584          # the Llama-8B MLP workload
