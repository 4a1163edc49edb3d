"""Host-side pieces of bench.py: the algorithmic bytes per step (the
numerators of every reported bandwidth and roofline fraction) against the
closed forms of the workloads, and the replica rule that keeps the timed
steps out of L2."""
import bench as B


def test_algorithmic_bytes_per_step():
    sb = B.step_bytes
    # c4a B=32 t=131072: 32 x 32736 keys x 256 B + 32 x (512 + 128) rows x 1024 B
    assert sb("c4a", 32, 131072, 0, 0) == 32 * 32736 * 256 + 32 * 640 * 1024 == 289_144_832
    # c128a B=8 t=131072: 8 x (1023 + 128) rows x 1024 B
    assert sb("c128a", 8, 131072, 0, 0) == 9_428_992
    # quantised c4a B=64 t=262144, fp8 / fp4 main cache, fp4 indexer keys (72 B)
    assert sb("c4a", 64, 262144, 1, 2) == 64 * 65504 * 72 + 64 * 640 * 516 == 322_977_792
    assert sb("c4a", 64, 262144, 2, 2) == 64 * 65504 * 72 + 64 * 640 * 288 == 313_638_912
    # quantised c128a B=64: 64 x (2047 + 128) rows of 516 / 288 / 580 B
    assert sb("c128a", 64, 262144, 1, 0) == 71_827_200
    assert sb("c128a", 64, 262144, 2, 0) == 40_089_600
    assert sb("c128a", 64, 262144, 3, 0) == 64 * 2175 * 580
    # a Reindex layer reads only its pool's keys
    assert sb("c4a", 32, 131072, 0, 0, pool=2048) == 32 * 2048 * 256 + 32 * 640 * 1024


def test_replicas_hold_four_l2():
    for name, spec in B.WORKLOADS.items():
        pool = spec[6] if len(spec) > 6 else 0
        r = B.replicas_for(spec[0], spec[1], spec[2], spec[4], spec[5], 2, pool)
        assert r >= 2 and r * B.step_bytes(spec[0], spec[1], spec[2], spec[4], spec[5], pool=pool) >= 4 * B.L2_BYTES, name


def test_flops_and_launch_counts():
    assert B.FMT_NAME[3] == "fp8+bf16rope" and B.ROW_BYTES[3] == 576 + 4


def test_ragged_lengths_are_seeded_and_bounded():
    a, b = B.ragged_lengths(32, 131072, 7), B.ragged_lengths(32, 131072, 7)
    assert (a == b).all() and a.min() >= 65536 and a.max() <= 131072


def test_reference_arm_times_the_steps_it_reports():
    """The oracle arm runs `warmup` + `steps` steps of the given workload (here
    a small one, whole steps) and prints the config it was handed unchanged."""
    import argparse
    args = argparse.Namespace(steps=2, warmup=1, gpus=1)
    cfg = {"workload": "tiny", "batch_per_gpu": 2}
    line = B.reference_arm(args, "c4a", 2, 4224, 4, cfg, "tiny")
    assert line["impl"] == "reference" and line["config"] is cfg
    assert line["steps"] == 2 and line["warmup"] == 1 and line["sequences_per_step"] == 2
    assert line["value"] > 0 and abs(line["ms_per_step"] * line["value"] - 1e3) < 1e-6 * 1e3
    dense = B.reference_arm(args, "c128a", 2, 128 * 40, 4, cfg, "tiny")
    assert dense["value"] > 0
