"""Pins for the oracle's number formats (E4M3, E2M1, unsigned E4M3, bf16).

The formats carry the FP8/FP4 index cache ('Token 的一生：DSV4 架构与 DSpark'
§3.1) and the FP8-latent / BF16-RoPE KV rows ('DeepSeek-V4 的交錯壓縮注意力
（CSA/HCA）', section '低精度與儲存策略的配合').  The pins are the formats'
textbook definitions: torch's own float8 / bfloat16 conversions as library
routines, exhaustive round trips, and hand-derived midpoint fixtures.
"""
import json
import os

import numpy as np
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_e4m3_decode_matches_torch_float8(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = orc.e4m3_table()
    nan = np.isnan(ref)
    assert (nan == np.isnan(mine)).all()
    assert nan.sum() == 2                      # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], mine[~nan])
    # signed zero kept
    assert np.signbit(mine[0x80]) and not np.signbit(mine[0x00])


def test_e4m3_round_trip_every_code(orc):
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert orc.e4m3_encode(orc.e4m3_value(c)) == c


def test_e4m3_midpoints_go_to_even(orc):
    for c in range(0, 0x7E):
        lo, hi = orc.e4m3_value(c), orc.e4m3_value(c + 1)
        mid = 0.5 * (lo + hi)
        even = c if c % 2 == 0 else c + 1
        assert orc.e4m3_encode(mid) == even
        assert orc.e4m3_encode(-mid) == 0x80 | even
        assert orc.e4m3_encode(np.nextafter(mid, 0.0)) == c
        assert orc.e4m3_encode(np.nextafter(mid, np.inf)) == c + 1


def test_e4m3_encode_matches_torch_in_range(orc):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(20000, generator=g) * torch.exp(torch.randn(20000, generator=g) * 3)).float()
    x = x[x.abs() < 440]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([orc.e4m3_encode(float(v)) for v in x.numpy()], dtype=np.uint8)
    assert np.array_equal(ref, mine)


def test_e4m3_saturates(orc):
    assert orc.e4m3_encode(448.0) == 0x7E
    assert orc.e4m3_encode(449.0) == 0x7E
    assert orc.e4m3_encode(1e30) == 0x7E
    assert orc.e4m3_encode(-1e30) == 0xFE


def test_e4m3_golden(orc):
    g = _gold("e4m3_points.json")
    for c, v in g["values"]:
        got = orc.e4m3_value(c)
        assert got == v and np.signbit(got) == np.signbit(v)
    for x, c in g["rounding"]:
        assert orc.e4m3_encode(x) == c, (x, c)


def test_e2m1_golden_and_round_trip(orc):
    g = _gold("e2m1_rounding.json")
    assert [orc.e2m1_value(c) for c in range(8)] == g["values"]
    assert [orc.e2m1_value(c | 8) for c in range(1, 8)] == [-v for v in g["values"][1:]]
    for x, c in g["rounding"]:
        assert orc.e2m1_encode(x) == c, (x, c)
    for c in range(16):
        assert orc.e2m1_encode(orc.e2m1_value(c)) == c


def test_ue4m3_is_positive_e4m3(orc):
    for c in range(0x7F):
        assert orc.ue4m3_value(c) == orc.e4m3_value(c) >= 0
        assert orc.ue4m3_encode(orc.ue4m3_value(c)) == c
    assert orc.ue4m3_encode(-3.0) == 0
    assert orc.ue4m3_encode(1e9) == 0x7E


def test_bf16_matches_torch_rne(orc):
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(50000, generator=g) * torch.exp(torch.randn(50000, generator=g) * 10)).float()
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1.00390625, 1.01171875, 3.3895e38, 1e-40])])
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mine = orc.bf16_encode_array(x.double().numpy())
    assert np.array_equal(ref, mine)
    back = orc.bf16_to_f64(mine)
    assert np.array_equal(back, x.to(torch.bfloat16).double().numpy())
