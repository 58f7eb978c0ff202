"""Host logic of the seeded workload module: shapes, parameter counts,
determinism of the generators.  CPU only."""
import numpy as np

import tables
from muon_optimizer_step_02_b200 import workloads as wl


def test_gpt11_matrix_set():
    """PR #1893 table "Architecture and training stack": 11 layers, 512d,
    8 query / 4 KV heads (head_dim 64), MLP 4x; 66 matrices (also the "66
    layers" of its GPTQ row)."""
    w = wl.workload(2)
    assert w.n_mats == 66
    assert w.numel() == 31_719_424
    assert set(w.shapes) == {(512, 512), (256, 512), (2048, 512), (512, 2048)}


def test_gpt11_ema_parameter_count():
    """Explicit tensor list of the EMA workload: 66 matrices + 8192x512 +
    4096x512 embeddings + 118 x 512 vectors + 92 scalars = 38,071,388; the
    1-D part is sized to the page's 34,401,372-parameter residual."""
    w = tables.workload(3)
    n = w.ema_numels()
    assert len(n) == 66 + 2 + 118 + 92
    assert sum(n) == 38_071_388
    assert 34_401_372 - 31_719_424 - 4096 * 512 - 4096 * 128 == 118 * 512 + 92


def test_large_configs():
    w4, w5 = wl.workload(4), wl.workload(5)
    assert w4.n_mats == 96 and w5.n_mats == 144
    assert (4096, 1024) in w4.shapes and (2048, 8192) in w5.shapes
    assert w5.numel() == 24 * (2 * 2048 * 2048 + 2 * 1024 * 2048
                               + 2 * 8192 * 2048)


def test_generators_are_seeded_and_independent():
    w = wl.workload(2)
    a = wl.grad_bits(w, 5, step=1)
    b = wl.grad_bits(w, 5, step=1)
    c = wl.grad_bits(w, 5, step=2)
    assert a.dtype == np.uint16 and a.shape == w.shapes[5]
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    g = wl.bf16_bits_to_f32(a)
    assert abs(float(np.std(g)) - 1e-3) < 5e-5
    W = wl.weight(w, 5)
    assert abs(float(np.std(W)) - 0.02) < 1e-3


def test_bf16_bits_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5],
                 dtype=np.float32)
    bits = wl.f32_to_bf16_bits(x)
    back = wl.bf16_bits_to_f32(bits)
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5]


def test_polar_express_table_is_an_input():
    t = tables.polar_express_k4()
    assert len(t) == 4 and all(len(r) == 3 for r in t)
    assert tables.workload(3).coeffs == [tuple(r) for r in t]
    # the package reads no table itself: workload 3 needs one passed in
    import pytest
    with pytest.raises(ValueError):
        wl.workload(3)
