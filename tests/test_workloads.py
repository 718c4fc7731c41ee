"""The seeded input generators: deterministic, right shapes, masks as the workloads state."""
import numpy as np
import torch

import workloads as WL


def test_cfg0_deterministic_and_shaped():
    a = WL.make_inputs(WL.CONFIGS["cfg0"], seed=0)
    b = WL.make_inputs(WL.CONFIGS["cfg0"], seed=0)
    c = WL.make_inputs(WL.CONFIGS["cfg0"], seed=1)
    assert a["H"].shape == (256, 256) and a["H"].dtype == torch.bfloat16
    assert a["W"].shape == (4096, 256) and a["W"].dtype == torch.bfloat16
    assert a["M"].shape == (1, 256) and a["M"].dtype == torch.uint8
    for key in ("H", "W", "M"):
        assert torch.equal(a[key], b[key])
    assert not torch.equal(a["H"], c["H"])
    assert 90 < int(a["M"].sum()) < 166          # Bernoulli(0.5) over 256 positions
    assert abs(float(a["W"].float().std()) - 0.02) < 0.002
    assert abs(float(a["H"].float().std()) - 1.0) < 0.02


def test_suffix_and_semi_ar_masks():
    m1 = WL.make_mask(WL.CONFIGS["cfg1"])
    assert int(m1.sum()) == 1024 and int(m1[0, 3071]) == 0 and int(m1[0, 3072]) == 1
    cfg4 = WL.CONFIGS["cfg4"]
    m4 = WL.make_mask(cfg4)
    per_seq = m4.sum(dim=1).tolist()
    assert per_seq == [7680 - 1024 * b for b in range(8)]
    assert int(m4.sum()) == 32768
    lo, hi = WL.make_windows(cfg4)
    assert lo.tolist() == [32 * (32 * b + 16) for b in range(8)]
    assert (hi - lo).tolist() == [32] * 8
    for b in range(8):     # the current block is fully masked, everything before it is not
        assert int(m4[b, lo[b]:hi[b]].sum()) == 32 and int(m4[b, :lo[b]].sum()) == 0


def test_cfg3_masks_nested_by_ratio():
    small = {r: WL.get_config(f"cfg3_r{r}", L=4096, d=8, V=16) for r in (0.1, 0.5, 0.9)}
    masks = {r: WL.make_inputs(c, seed=0)["M"] for r, c in small.items()}
    assert torch.all(masks[0.1] <= masks[0.5]) and torch.all(masks[0.5] <= masks[0.9])


def test_sample_rows():
    s = WL.sample_rows(10_000, 512, seed=0)
    assert s.size == 512 and np.all(np.diff(s) > 0) and s[-1] < 10_000
    assert np.array_equal(s, WL.sample_rows(10_000, 512, seed=0))
    assert np.array_equal(WL.sample_rows(100, 512), np.arange(100))


def test_bf16_bits_roundtrip():
    t = torch.tensor([1.0, -2.5, 0.0078125, 3.0e38]).to(torch.bfloat16)
    bits = WL.bf16_bits(t)
    assert bits.dtype == np.uint16
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    assert torch.equal(back, t)


def test_sweep_matches_individual_draws():
    names = ["cfg3_r0.1", "cfg3_r0.9"]
    small = {n: WL.get_config(n, L=512, d=8, V=16) for n in names}
    WL.CONFIGS.update({f"_t_{n}": c for n, c in small.items()})
    try:
        sweep = WL.make_sweep_inputs([f"_t_{n}" for n in names], seed=3)
        for n in names:
            one = WL.make_inputs(small[n], seed=3)
            got = sweep[small[n].name]
            for key in ("H", "W", "M"):
                assert torch.equal(one[key], got[key])
    finally:
        for n in names:
            WL.CONFIGS.pop(f"_t_{n}")
