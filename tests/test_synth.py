"""The seeded input generator: SplitMix64 against its published sequence, normal draws, determinism."""
import numpy as np

import synth


def test_splitmix64_published_sequence():
    # SplitMix64 from seed 1234567 (the sequence printed with Vigna's reference implementation)
    ref = [6457827717110365317, 3203168211198807973, 9817491932198370423, 4593380528125082431,
           16408922859458223821]
    assert synth.splitmix64_sequence(1234567, 5).tolist() == ref


def test_counter_based_slices_agree():
    a = synth.normal_f32(5, 3, 7, 1000, 0.0, 1.0)
    b = synth.normal_f32(5, 3, 7, 400, 0.0, 1.0, offset=600)
    np.testing.assert_array_equal(a[600:], b)
    c = synth.normal_f32(5, 3, 7, 1000, 0.0, 1.0, nthreads=4)
    np.testing.assert_array_equal(a, c)
    assert not np.array_equal(a, synth.normal_f32(5, 3, 8, 1000, 0.0, 1.0))


def test_normal_moments():
    z = synth.normal_f32(0, 1, 0, 400_000, 0.0, 1.0).astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    assert abs(np.mean(np.abs(z) > 2) - 0.0455) < 0.003
    w = synth.normal_f32(0, 6, 0, 100_000, 0.0, 0.02)
    assert abs(w.std() - 0.02) < 5e-4


def test_bf16_rows_and_redraw():
    cfg = synth.CONFIGS["tiny"]
    x = synth.hidden(cfg)
    assert x.shape == (cfg.T, cfg.d) and x.dtype == np.uint16
    r = synth.hidden_rows(cfg, [3, 5])
    np.testing.assert_array_equal(r, x[[3, 5]])
    r1 = synth.hidden_rows(cfg, [3], [1])
    assert not np.array_equal(r1[0], x[3])
    f = synth.bf16_to_f32(x)
    assert abs(float(f.std()) - 1) < 0.1


def test_zipf_bias_skews_popularity():
    cfg = synth.CONFIGS["skew_120b"]
    ranks = synth.zipf_ranks(cfg)
    assert sorted(ranks.tolist()) == list(range(1, cfg.E + 1))
    b = synth.router_bias(cfg).astype(np.float64)
    p = np.exp(b - b.max())
    p /= p.sum()
    top = p[np.argmin(ranks)]
    assert 0.2 < top < 0.35  # Zipf(1.2) over 128 experts: the top expert holds ~27% of the mass


def test_configs_match_workloads():
    c = synth.CONFIGS
    assert (c["tiny"].T, c["tiny"].d, c["tiny"].I, c["tiny"].E, c["tiny"].k) == (32, 128, 128, 4, 2)
    assert (c["decode_20b"].T, c["decode_20b"].E, c["decode_20b"].k) == (16, 32, 4)
    assert (c["prefill_20b"].T, c["prefill_20b"].E) == (4096, 32)
    assert (c["moe_120b"].T, c["moe_120b"].E) == (8192, 128)
    assert (c["skew_120b"].T, c["skew_120b"].E, c["skew_120b"].zipf_s) == (16384, 128, 1.2)
    for name in ("decode_20b", "prefill_20b", "moe_120b", "skew_120b"):
        assert c[name].d == c[name].I == 2880 and c[name].k == 4
