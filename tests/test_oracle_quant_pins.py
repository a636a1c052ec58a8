"""Pins for the oracle's per-token FP8 quantisation (CPU only).

What is fixed independently of the oracle's code:
- the e4m3 encoding is the inverse of the OCP decoding on every finite code,
  rounds halfway cases to the even code and saturates at 448 (the OCP
  definition; torch's float8_e4m3fn cast is a second, independent encoder);
- the scale is absmax / 448 in fp32 (so the largest element maps to +-448) and
  an all-zero row gets scale 1;
- the fused column order only permutes the output columns (the scale is a
  per-row maximum, which no permutation changes).
"""
import numpy as np
import pytest
import torch

import oracle


def bf16_bits(x):
    """float32 values -> bf16 bit patterns (round to nearest even, torch's cast)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def torch_quantize(bits):
    """Per-row absmax quantisation written with torch's own e4m3 cast."""
    x = bf16_values(bits)
    amax = np.max(np.abs(x), axis=1)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    t = (torch.from_numpy(x) / torch.from_numpy(s)[:, None]).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy(), s


def test_every_finite_code_round_trips():
    table = oracle.e4m3_table()
    codes = [c for c in range(256) if (c & 0x7F) != 0x7F]
    vals = np.array([table[c] for c in codes], np.float32)
    # a leading 448 makes the row's scale exactly 1, so the codes are encode(value)
    row = np.concatenate([[448.0], vals]).astype(np.float32)[None, :]
    pad = (-row.shape[1]) % 16
    row = np.concatenate([row, np.zeros((1, pad), np.float32)], axis=1)
    q, s = oracle.quantize(bf16_bits(row))
    assert s[0] == np.float32(1.0)
    assert q[0, 0] == 0x7E
    got = q[0, 1:1 + len(codes)]
    want = np.array(codes, np.uint8)
    want[want == 0x80] = 0x80  # -0 keeps its sign
    assert np.array_equal(got, want)


def test_halfway_values_round_to_the_even_code_and_match_torch():
    table = oracle.e4m3_table()
    mids, even = [], []
    for c in range(0, 0x7E):
        a, b = table[c], table[c + 1]
        mids.append((a + b) / 2)
        even.append(c if c % 2 == 0 else c + 1)
    mids = np.array(mids, np.float32)
    row = np.concatenate([[448.0], mids, -mids]).astype(np.float32)
    row = np.concatenate([row, np.zeros((-row.size) % 16, np.float32)])[None, :]
    bits = bf16_bits(row)
    assert np.array_equal(bf16_values(bits), row)  # every midpoint is exact in bf16
    q, _ = oracle.quantize(bits)
    n = len(mids)
    assert np.array_equal(q[0, 1:1 + n], np.array(even, np.uint8))
    assert np.array_equal(q[0, 1 + n:1 + 2 * n], np.array(even, np.uint8) | 0x80)
    tq, _ = torch_quantize(bits)
    assert np.array_equal(q, tq)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_rows_match_torch_cast(seed):
    g = np.random.default_rng(seed)
    M, K = 7, 512
    x = g.standard_normal((M, K)).astype(np.float32) * np.float32(10.0) ** g.integers(-6, 6, size=(M, 1))
    x[2, :] = 0.0                          # all-zero row
    x[3, 5] = 1e4                          # one outlier dominates the scale
    x[4, :] = np.float32(1e-30) * np.sign(x[4, :])  # tiny values: subnormal and zero codes
    bits = bf16_bits(x)
    q, s = oracle.quantize(bits)
    tq, ts = torch_quantize(bits)
    assert np.array_equal(s, ts)
    assert np.array_equal(q, tq)
    assert s[2] == 1.0 and not q[2].any()
    # the largest magnitude of each nonzero row maps to +-448
    for m in (0, 1, 3, 5, 6):
        k = int(np.argmax(np.abs(bf16_values(bits[m]))))
        assert q[m, k] & 0x7F == 0x7E


def test_order_only_permutes_columns():
    g = np.random.default_rng(5)
    M, K, Kd = 5, 256, 48
    bits = bf16_bits(g.standard_normal((M, K)).astype(np.float32))
    dense_idx = np.sort(g.choice(K, Kd, replace=False)).astype(np.int32)
    q0, s0 = oracle.quantize(bits)
    q1, s1 = oracle.quantize(bits, dense_idx=dense_idx)
    sparse = np.setdiff1d(np.arange(K), dense_idx)
    order = np.concatenate([sparse, dense_idx])
    assert np.array_equal(s0, s1)
    assert np.array_equal(q1, q0[:, order])


def test_rejects_a_bad_dense_set():
    bits = np.zeros((1, 32), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.quantize(bits, dense_idx=np.array([5, 3], np.int32))
