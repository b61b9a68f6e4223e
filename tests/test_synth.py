"""The seeded input generator: distribution, encodings (against torch's conversions), determinism."""
import numpy as np
import torch

from lsa_synth import gen
from lsa_synth import workloads as W


def test_normal_draws_moments_and_grid():
    key = gen.tensor_key(0, 1)
    x = gen.normal_f32(key, np.arange(1 << 20, dtype=np.uint64)).astype(np.float64)
    n = x.size
    assert abs(x.mean()) < 5 / np.sqrt(n)
    assert abs(x.var() - 1.0) < 5 * np.sqrt(2.0 / n)
    assert np.abs(x).max() <= 6.0
    assert np.all(x * 2 ** 17 == np.round(x * 2 ** 17))             # exact multiples of 2**-17
    # Irwin-Hall(12) kurtosis is 3 - 1.2/12 = 2.9
    assert abs(((x - x.mean()) ** 4).mean() / x.var() ** 2 - 2.9) < 0.02


def test_draws_are_pure_functions_of_counter():
    key = gen.tensor_key(3, 16)
    a = gen.normal_f32(key, np.arange(1000, 2000, dtype=np.uint64))
    b = gen.normal_f32(key, np.arange(0, 3000, dtype=np.uint64))[1000:2000]
    assert np.array_equal(a, b)
    assert not np.array_equal(a, gen.normal_f32(gen.tensor_key(4, 16), np.arange(1000, 2000, dtype=np.uint64)))
    u = gen.uniform_f32(key, np.arange(1 << 16, dtype=np.uint64))
    assert u.min() >= 0 and u.max() < 1 and abs(u.mean() - 0.5) < 0.01


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = (rng.normal(size=100000) * 10.0 ** rng.integers(-20, 20, size=100000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(gen.f32_to_bf16_bits(x), ref)


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-448, 448, size=50000), rng.normal(size=50000) * 2.0 ** -7,
                        np.array([0.0, 448.0, -448.0, 2 ** -10, -(2 ** -10), 1.0625, 1.1875])]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = gen.f32_to_e4m3(x)
    assert np.array_equal(mine, ref)


def test_row_quantisation_error_bound():
    key = gen.tensor_key(1, 1)
    x = gen.normal_f32(key, gen.cache_ctr(0, np.arange(200), 128))
    codes, scale = gen.quantize_rows_e4m3(x)
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy() * scale[:, None]
    amax = np.abs(x).max(axis=1)
    assert np.allclose(np.abs(dec).max(axis=1), amax, rtol=2 ** -4)
    # relative error of e4m3 rounding is at most 2**-4 for normal codes; absolute floor for subnormals
    err = np.abs(dec - x)
    assert np.all(err <= np.maximum(np.abs(x) * 2 ** -4, scale[:, None] * 2 ** -10) * (1 + 1e-6))


def test_choose_without_replacement():
    p = gen.choose_without_replacement(0, gen.TID_PLANT, 0, 4096, 41)
    assert p.size == 41 and len(set(p.tolist())) == 41 and np.all(np.diff(p) > 0)
    assert p.min() >= 0 and p.max() < 4096
    assert np.array_equal(p, gen.choose_without_replacement(0, gen.TID_PLANT, 0, 4096, 41))


def test_workload_lengths_and_positions():
    w = W.WORKLOADS["decode_cli_128k"]
    L = W.lengths(w)
    assert L.shape == (32,) and L.min() >= 65536 and L.max() <= 131072 and len(set(L.tolist())) > 20
    q_seq, q_pos = W.query_rows(w, w.passes[0])
    assert np.array_equal(q_pos, L - 1) and np.array_equal(q_seq, np.arange(32))
    w5 = W.WORKLOADS["mtp_256k"]
    q_seq, q_pos = W.query_rows(w5, w5.passes[0])
    assert q_pos[:4].tolist() == [262140, 262141, 262142, 262143] and q_seq.size == 256
    w2 = W.WORKLOADS["prefill_32k"]
    _, q_pos = W.query_rows(w2, w2.passes[0])
    assert q_pos[0] == 30720 and q_pos[-1] == 32767
    assert w5.queries_per_step() == 64 * 7


def test_plant_plan():
    w = W.WORKLOADS["tiny_decode"]
    rows, dirs = W.plant_plan(w, w.passes[0])
    assert rows[0].size == 41
    assert abs(np.linalg.norm(dirs[0]) - 8.0) < 1e-5           # sqrt(64)
    w4 = W.scaled("decode_hi_1m", len_lo=8192, len_hi=8192)
    rows, _ = W.plant_plan(w4, w4.passes[0])
    assert all(r.size == 16 * 64 for r in rows)
    assert all(np.unique(r // 64).size == 16 for r in rows)
