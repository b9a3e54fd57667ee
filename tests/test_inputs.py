"""The seeded input generator (CPU): the published SplitMix64 sequence,
chunking and offset independence, the bf16 rounding, the normal deviates'
distribution, and the workload recipes."""
import numpy as np
import torch

from routing_grouped_gemm_moe_b200 import inputs as I


def test_splitmix64_matches_the_published_sequence():
    """SplitMix64 seeded with 0 (Steele, Lea & Flood; the reference
    generator's first three outputs)."""
    b = I.random_bits(0, 0, 3, "cpu")
    got = [int(x) & (2 ** 64 - 1) for x in b]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    # the scalar mixer (used for stream keys) is the same function
    assert I._mix_int(0x9E3779B97F4A7C15) == 0xE220A8397B1DCDAF


def test_draws_do_not_depend_on_chunking_or_offset():
    key = I.stream_key(7, 3)
    whole = I.normal_bf16(key, (1000, 24), 0.5)
    chunked = I.normal_bf16(key, (1000, 24), 0.5, chunk=4096)
    assert torch.equal(whole.view(torch.int16), chunked.view(torch.int16))
    tail = I.normal_bf16(key, (500, 24), 0.5, start=500 * 24)
    assert torch.equal(whole[500:].view(torch.int16), tail.view(torch.int16))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    v = torch.from_numpy(rng.standard_normal(100000).astype(np.float32) * 7)
    v[:16] = torch.tensor([0.0, -0.0, 1.0, -1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 3.0e38, -3.0e38,
                           1e-40, -1e-40, 2 ** -126, 65504.0, 1.00390625, 1.01171875, 0.5, -0.75])
    ours = I.f32_to_bf16_bits(v)
    ref = v.to(torch.bfloat16).view(torch.int16)
    assert torch.equal(ours, ref)


def test_normal_deviates_distribution():
    x = I.normal_f64(I.stream_key(11, 1), 0, 1 << 20).numpy()
    assert abs(x.mean()) < 3e-3
    assert abs(x.std() - 1.0) < 3e-3
    assert np.abs(x).max() < 4.5                       # tails cut near 4.3 sigma
    # the quantile table reproduces the normal CDF at a few points
    for z, p in ((-1.0, 0.158655), (0.0, 0.5), (1.645, 0.95)):
        assert abs(np.mean(x < z) - p) < 2e-3


def test_skewed_logits_recipe():
    cfg = I.CONFIGS["skewed"]
    bias = I.zipf_bias(cfg).numpy()
    empty = np.nonzero(bias <= -1e3)[0]
    assert len(empty) == 4
    ranks = np.sort(-bias[bias > -1e3]) / 1.2          # ln r for r = 1..60
    assert np.allclose(np.exp(ranks), np.arange(1, 61), rtol=1e-6)
    lg = I.make_logits(cfg, rows=range(256))
    idx = torch.topk(lg, cfg.k, dim=1).indices
    assert not np.isin(idx.numpy(), empty).any()       # the four experts get no tokens


def test_workloads_have_the_benchmark_shapes():
    shapes = {n: (c.T, c.d, c.E, c.k, c.f) for n, c in I.CONFIGS.items()}
    assert shapes["tiny"] == (256, 128, 8, 2, 256)
    assert shapes["fine"] == (4096, 2048, 32, 4, 1024)
    assert {shapes[f"pool_e{e}"] for e in (8, 32, 128)} == {(16384, 2048, e, 4, 1024) for e in (8, 32, 128)}
    assert shapes["skewed"] == (8192, 4096, 64, 8, 1536)
    assert shapes["large"] == shapes["large_bf16"] == (32768, 4096, 128, 8, 2048)
    assert I.CONFIGS["large"].dtype == "mxfp8" and I.CONFIGS["large_bf16"].dtype == "bf16"
    assert I.CONFIGS["tiny"].router == "proj" and I.CONFIGS["fine"].router == "proj"
