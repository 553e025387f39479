"""The seeded input generators: shapes, value ranges and determinism.

The generators feed both the CUDA path and the oracle, so a generator that
emitted an out-of-contract value (a NaN E4M3 code, an E8M0 byte of 255, an
offset run that does not match the counts) would make both sides agree on
garbage.  CPU only.
"""
import numpy as np
import torch

from combine_moe_update_b200 import inputs as gen


def test_gmm_inputs_shapes_ranges_and_seed():
    counts = [3, 0, 17, 130]
    a = gen.gmm_inputs(5, counts, 1024, 48, spare_rows=2)
    b = gen.gmm_inputs(5, counts, 1024, 48, spare_rows=2)
    assert a.expand_x.shape == (152, 1024) and a.weight.shape == (4, 48, 1024)
    np.testing.assert_array_equal(a.offsets, [0, 3, 3, 20, 150])
    assert a.expand_x.min() >= -127 and a.weight.min() >= -128
    assert (a.dyn_scales > 0).all() and (a.weight_scales > 0).all()
    np.testing.assert_array_equal(a.expand_x, b.expand_x)
    np.testing.assert_array_equal(a.weight, b.weight)
    one = gen.gmm_inputs(5, counts, 1024, 48, one_hot=True)
    assert ((one.expand_x != 0).sum(axis=1) <= 1).all()
    assert np.abs(one.weight).max() <= 15 and (one.dyn_scales == 1).all()


def test_gmm_inputs_mx_codes_are_finite():
    g = gen.gmm_inputs_mx(6, [40, 0, 9], 1024, 64, spare_rows=1)
    for codes in (g.expand_x, g.weight):
        assert not np.isin(codes, [0x7F, 0xFF]).any()  # S.1111.111 is NaN in E4M3
    assert g.x_sf.shape == (50, 32) and g.weight_sf.shape == (3, 64, 32)
    for sf in (g.x_sf, g.weight_sf):
        assert sf.min() >= 117 and sf.max() <= 137  # never the E8M0 NaN byte 255
    # every finite code is reachable
    assert len(np.unique(g.weight)) == 254


def test_device_weight_generators_on_cpu():
    w, ws = gen.gmm_weights_device(3, 2, 16, 256, "cpu")
    assert w.dtype == torch.int8 and w.shape == (2, 16, 256) and ws.shape == (2, 16)
    assert float(ws.min()) >= 1e-4 and float(ws.max()) <= 1e-3
    wm, sf = gen.gmm_weights_device_mx(3, 2, 16, 256, "cpu")
    assert wm.dtype == torch.uint8 and sf.shape == (2, 16, 8)
    codes = wm.numpy()
    assert not np.isin(codes, [0x7F, 0xFF]).any()
    assert int(sf.min()) >= 117 and int(sf.max()) <= 137
    w2, _ = gen.gmm_weights_device(3, 2, 16, 256, "cpu")
    assert torch.equal(w, w2)


def test_host_weight_generators_match_the_device_distribution():
    hw = gen.gmm_weights_host(4, [0, 5], 32, 256)
    assert set(hw) == {0, 5} and hw[5][0].shape == (32, 256) and hw[5][1].shape == (32,)
    hm = gen.gmm_weights_host_mx(4, [1], 32, 256)
    codes, sf = hm[1]
    assert sf.shape == (32, 8) and not np.isin(codes, [0x7F, 0xFF]).any()


def test_expert_workloads_carry_their_matmul_parameters():
    for name, mode in (("deepseek_decode_bs512_expert", 2), ("deepseek_decode_bs512_expert_mx", 4),
                       ("expert_e32_bs128", 2), ("expert_e32_bs128_mx", 4)):
        w = gen.make(name, bs=8)
        assert w.quant_mode == mode
        assert w.meta["expert_out_dim"] == w.hidden and "weight_seed" in w.meta
