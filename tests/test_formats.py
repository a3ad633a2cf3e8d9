"""Pins for the oracle's number-format decoders and the input generator's
encoders. Each decoder is checked against something other than itself: the
e4m3 and bf16 decoders against torch's own casts (an independent library
implementation), the e2m1 decoder against the value table of the OCP MX
e2m1 format, restated here by hand."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def test_e4m3_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        got = oracle.e4m3_to_double(c)
        want = float(ref[c])
        if math.isnan(want):
            assert math.isnan(got), c
        else:
            assert got == want, (c, got, want)


def test_decode_tables_hold_the_decoders_values():
    """The logits loops read decoded values from tables filled by the decoders;
    every entry must be exactly the decoder's value (NaN where it is NaN), and
    the e4m3 table is also checked against torch directly."""
    e4, e2 = oracle.decode_tables()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        got, want = e4[c], oracle.e4m3_to_double(c)
        if math.isnan(want):
            assert math.isnan(got) and math.isnan(float(ref[c])), c
        else:
            assert got == want == float(ref[c]), c
    e2m1 = [0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6]
    for c in range(16):
        assert e2[c] == oracle.e2m1_to_double(c) == e2m1[c], c
        assert math.copysign(1.0, e2[c]) == math.copysign(1.0, e2m1[c]), c


def test_e4m3_landmarks():
    # max normal, min normal, min subnormal, one, negative zero
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_double(0x38) == 1.0
    assert oracle.e4m3_to_double(0x80) == 0.0
    assert math.isnan(oracle.e4m3_to_double(0x7F))
    assert math.isnan(oracle.e4m3_to_double(0xFF))


# OCP Microscaling spec, FP4 E2M1 value table (code -> value).
E2M1_TABLE = {0b0000: 0.0, 0b0001: 0.5, 0b0010: 1.0, 0b0011: 1.5,
              0b0100: 2.0, 0b0101: 3.0, 0b0110: 4.0, 0b0111: 6.0,
              0b1000: -0.0, 0b1001: -0.5, 0b1010: -1.0, 0b1011: -1.5,
              0b1100: -2.0, 0b1101: -3.0, 0b1110: -4.0, 0b1111: -6.0}


def test_e2m1_all_codes_match_format_table():
    for c, v in E2M1_TABLE.items():
        assert oracle.e2m1_to_double(c) == v, c


def test_bf16_matches_torch():
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    rng = np.random.default_rng(0)
    for b in list(rng.integers(0, 65536, 4000)) + [0x0000, 0x8000, 0x3F80, 0x7F7F, 0x0001, 0x7F80]:
        got = oracle.bf16_to_double(int(b))
        want = ref[int(b)]
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want, hex(int(b))


def test_e2m1_quantiser_rounds_to_nearest_even():
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    # exact grid values round-trip
    x = torch.tensor(list(grid) + list(-grid[1:]), dtype=torch.float32)
    codes = workloads.quantize_e2m1_rne(x)
    back = [E2M1_TABLE[int(c)] for c in codes]
    assert back == list(x.numpy())
    # midpoints go to the code with an even mantissa bit
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=torch.float32)
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    got = [E2M1_TABLE[int(c)] for c in workloads.quantize_e2m1_rne(mids)]
    assert got == want
    # saturation and nearest
    got = [E2M1_TABLE[int(c)] for c in workloads.quantize_e2m1_rne(
        torch.tensor([100.0, -7.0, 0.26, 2.6, -0.74], dtype=torch.float32))]
    assert got == [6.0, -6.0, 0.5, 3.0, -0.5]


@pytest.mark.parametrize("name", ["tiny", "decode", "fp4"])
def test_generator_is_deterministic(name):
    a = workloads.make_config(name)
    b = workloads.make_config(name)
    for f in ("q", "kv_cache", "block_table", "context_lens", "weights"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f


def test_generator_shapes_and_recipe():
    wl = workloads.make_config("decode")
    assert wl.q.shape == (64, 1, 64, 128) and wl.q.dtype == torch.uint8
    ctx = wl.context_lens
    assert int(ctx.min()) >= 1024 and int(ctx.max()) <= 8192
    # each row's used block-table slots are distinct pages of one shuffled pool
    used = torch.cat([wl.block_table[b, :(int(ctx[b]) + 63) // 64] for b in range(wl.B)])
    assert used.unique().numel() == used.numel() == wl.num_pages
    # scales in [0.5, 2]
    s = wl.kv_cache[:, 64 * 128:].contiguous().view(torch.float32)
    assert float(s.min()) >= 0.5 and float(s.max()) <= 2.0
    st = workloads.make_config("stress")
    c = st.context_lens
    assert int((c == 0).sum()) >= st.B // 10
    assert int(c.max()) <= 4096
