"""The hand-built edge inputs are what the edge-case parity tests say they are (CPU, via the oracle)."""
import numpy as np

from oracle import oracle_c as OC
from oracle import oracle_np as ON
from tests import edge_inputs as E

N, K = 60, 512
SLOTS = (np.arange(K) % 16) == E.OUT_SLOT


def test_int4_edge_categories():
    w = E.int4_edge(N, K, seed=1)
    cat = w["cat"]
    wf = OC.int4_dequant(*OC.int4_pack(w["q"], w["sc"], w["zc"], w["ss"], w["zs"]))
    assert np.all(np.isin(w["sc"][cat == 1], (0, 255))) and np.all(np.isin(w["zc"][cat == 1], (0, 255)))
    assert np.all((w["ss"][cat == 2] & 0x7C00) == 0) and np.all(w["ss"][cat == 2] != 0)
    assert np.any((w["ss"][cat == 3] & 0x7FFF) == 0) and np.any((w["zs"][cat == 3] & 0x7FFF) == 0)
    assert np.all(wf[cat == 4][:, SLOTS] == 0.0) and np.all(wf[cat == 4][:, ~SLOTS][::7] == wf[cat == 4][:, ~SLOTS][::7])
    assert np.count_nonzero(wf[cat == 4][:, ~SLOTS]) > 0.8 * wf[cat == 4][:, ~SLOTS].size
    assert np.any(w["ss"][cat == 5] & 0x8000) and np.any(w["zs"][cat == 5] & 0x8000)
    assert np.all(np.isfinite(wf))


def test_int6_edge_categories():
    w = E.int6_edge(N, K, seed=2)
    cat = w["cat"]
    wf = OC.int6_dequant(*OC.int6_pack(w["q"], w["sc"], w["st"]))
    assert set(np.unique(w["sc"][cat == 1])) == {-128, -127, 127}
    assert np.all((w["st"][cat == 2] & 0x7C00) == 0)
    assert np.any(w["st"][cat == 3] == 0) and np.any(w["sc"][cat == 3] == 0)
    assert np.all(wf[cat == 4][:, SLOTS] == 0.0)
    assert np.any(w["st"][cat == 5] & 0x8000)
    assert np.all(np.isfinite(wf))


def test_affine_edge_categories():
    for bits, G in ((2, 64), (4, 32), (8, 128)):
        w = E.affine_edge(N, K, bits, G, seed=3)
        cat = w["cat"]
        wf = OC.affine_dequant(*OC.affine_pack(w["q"], w["s"], w["b"], bits, G), bits, G)
        assert np.all((w["s"][cat == 1] & 0x7FFF) == 0)
        assert np.all(ON.f32_from_bf16_bits(w["s"][cat == 2]) < 0) and np.all(ON.f32_from_bf16_bits(w["b"][cat == 2]) < 0)
        assert np.all((w["s"][cat == 3] & 0x7F80) == 0) and np.all((w["b"][cat == 3] & 0x7F80) == 0)
        assert np.all(wf[cat == 4][:, SLOTS] == 0.0)
        assert np.all(np.abs(ON.f32_from_bf16_bits(w["s"][cat == 5])) >= 2.0 ** 8 * 0.99)
        assert np.all(np.isfinite(wf))


def test_activation_kinds():
    x = {k: ON.f32_from_bf16_bits(E.activation(k, K, seed=4)).astype(np.float64) for k in E.X_KINDS}
    for kind, ratio in (("outlier10", 2.0 ** 10), ("outlier7", 2.0 ** 7)):
        blocks = np.abs(x[kind].reshape(-1, 16))
        others = np.delete(blocks, E.OUT_SLOT, axis=1).max(axis=1)
        assert np.allclose(blocks[:, E.OUT_SLOT] / others, ratio, rtol=2 ** -7)
    sub = E.activation("subnormal", K, seed=4)
    assert np.all((sub & 0x7F80) == 0) and np.all((sub & 0x7F) != 0)
    zg = x["zero_grp"].reshape(-1, 32)
    assert np.any(np.all(zg == 0, axis=1)) and np.any(np.all(zg != 0, axis=1))
    ms = E.activation("mixed_sub", K, seed=4)
    assert np.all((ms[3::4] & 0x7F80) == 0) and np.all((ms[0::4] & 0x7F80) != 0)
    assert np.all(np.abs(x["wide20"][SLOTS]) == 2.0 ** 20)
