"""Host-side arithmetic of bench.py (CPU): the algorithmic work per
token-head behind the roofline fractions, and the per-rank seeds."""
import bench


def test_algorithmic_work_per_token_head():
    # Pythia-shaped prefill: d = dv = 256, p = 128, F = 256
    flops_featmap, flops_scan, bytes_fused = bench.algorithmic_per_token_head(256, 256, 128, 256)
    assert flops_featmap == 2 * (2 * 256 * 128) == 131072           # two Hedgehog projections
    assert flops_scan == 4 * 256 * (256 + 1) == 263168              # numerator and denominator, update + readout
    assert flops_featmap + flops_scan == 394240
    assert bytes_fused == 2 * (256 + 256 + 256) + 4 + 2 * 256 == 2052   # q, k, v in, dt in, o out


def test_rank_seeds_are_distinct_and_rank0_keeps_the_base():
    seeds = [bench.rank_seed(1, r) for r in range(8)]
    assert seeds[0] == 1
    assert len(set(seeds)) == 8
