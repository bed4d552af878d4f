"""The small-M path's NF4 reading ("level": bf16_rne(level) * absmax) is no
less faithful to the exact decode (level * absmax) than the tcgen05 path's
("product": bf16_rne(fp32(level * absmax))). The "grouped-nf4-gemm" README's
measured table compares fidelity of the fused path against dequantise-to-bf16;
here the two bf16 placements are compared with the exact value, on weights
and on layer outputs (oracle/nf4_fidelity.py)."""

from oracle import nf4_fidelity as fid


def test_level_weights_no_less_faithful_than_product():
    e = fid.weight_errors()
    assert e["level"]["rel_rms"] <= e["product"]["rel_rms"]
    assert e["level"]["rel_max"] <= e["product"]["rel_max"]
    # both are one bf16 rounding at most (2^-8 relative)
    for m in fid.MODES:
        assert e[m]["rel_max"] <= 2.0 ** -8 * (1 + 2.0 ** -20)


def test_level_layer_no_less_faithful_on_block_scale_data():
    e = fid.layer_errors(3, 256, 320, 40, 2, seed=42, std_gu=0.06, std_dn=0.06, spread=True)
    assert e["rms_y"] > 1.0
    assert e["level"]["rel_rmse"] <= e["product"]["rel_rmse"]
    assert e["level"]["max_scaled"] <= e["product"]["max_scaled"]


def test_level_layer_no_less_faithful_on_unit_scale_layer():
    e = fid.layer_errors(8, 256, 512, 64, 2, seed=7, std_gu=1.5 / 16, std_dn=2.0 / 512 ** 0.5)
    assert e["rms_y"] > 1.0
    assert e["level"]["rel_rmse"] <= e["product"]["rel_rmse"]
