"""Host-side logic on the CPU: the seeded input recipe of the five workloads,
the bf16 helpers, and the bench's byte accounting and input-ring sizing.

None of this is verification arithmetic; it decides what the parity tests
and the bench feed to the kernels and how the bench turns a time into a
roofline fraction, so a mistake here would silently change every measured
number.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import bench
import workloads


# ----------------------------------------------------------- input recipe
@pytest.mark.parametrize("cfg", workloads.CONFIGS, ids=lambda c: c.name)
def test_step_shapes_dtypes_and_determinism(cfg):
    B = min(cfg.B, 3)
    a = workloads.make_step(cfg, 7, B=B)
    b = workloads.make_step(cfg, 7, B=B)
    c = workloads.make_step(cfg, 8, B=B)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    assert a.target.shape == (B, cfg.gamma + 1, cfg.V) and a.target.dtype == dt
    assert a.draft.shape == (B, cfg.gamma, cfg.V) and a.draft.dtype == dt
    assert a.target.is_contiguous() and a.draft.is_contiguous()
    want_tok = (B, cfg.K, cfg.gamma) if cfg.multidraft else (B, cfg.gamma)
    assert tuple(a.tokens.shape) == want_tok and a.tokens.dtype == torch.int32
    assert int(a.tokens.min()) >= 0 and int(a.tokens.max()) < cfg.V
    assert a.temps.shape == (B,) and a.temps.dtype == torch.float32
    # same (config, step) -> identical bits; another step -> other inputs
    assert torch.equal(a.target, b.target) and torch.equal(a.draft, b.draft)
    assert torch.equal(a.tokens, b.tokens)
    assert not torch.equal(a.target, c.target)
    assert torch.isfinite(a.target.float()).all() and torch.isfinite(a.draft.float()).all()


def test_temperature_schedules():
    t1 = workloads.temperatures(workloads.get(1)).numpy()
    assert np.array_equal(t1, np.array([0.7 if b % 2 == 0 else 1.0 for b in range(16)], np.float32))
    t3 = workloads.temperatures(workloads.get(3)).numpy()
    assert np.allclose(t3, [(0.1, 0.4, 0.7)[b % 3] for b in range(8)])
    t4 = workloads.temperatures(workloads.get(4)).numpy()
    assert t4.shape == (256,)
    assert set(t4.tolist()) <= set(np.array([0.0, 0.1, 0.4, 0.7, 1.0], np.float32).tolist())
    assert (t4 == 0.0).any() and (t4 > 0.0).any()  # both greedy and sampled rows
    # drawn once: the same schedule at every call (and so at every step)
    assert np.array_equal(t4, workloads.temperatures(workloads.get(4)).numpy())
    for i in (0, 2):
        assert np.all(workloads.temperatures(workloads.get(i)).numpy() == 1.0)


def test_value_distributions_follow_the_recipe():
    # C0: target ~ N(0, 2.0), draft - target ~ N(0, 0.5) (fp32, exact)
    s0 = workloads.make_step(0, 0)
    assert abs(float(s0.target.std()) - 2.0) < 0.05
    assert abs(float((s0.draft - s0.target[:, :4]).std()) - 0.5) < 0.02
    # C2: draft = 0.8 target + N(0, 1.0): regression slope 0.8
    s2 = workloads.make_step(2, 0, B=1)
    t = s2.target[:, :8].float().flatten()
    d = s2.draft.float().flatten()
    slope = float((t * d).mean() / (t * t).mean())
    assert abs(slope - 0.8) < 0.02
    assert abs(float(s2.target.float().std()) - 2.5) < 0.05
    # C4: the mean logit falls as -1.1 ln(v + 1) over token ids
    s4 = workloads.make_step(4, 0, B=2)
    z = s4.target.float()
    lo = float(z[..., 1000:2000].mean())
    hi = float(z[..., 100000:101000].mean())
    want = -1.1 * (np.log(100500.0) - np.log(1500.0))
    assert abs((hi - lo) - want) < 0.3


def test_greedy_rows_draw_the_draft_argmax():
    st = workloads.make_custom(4, 3, 257, dtype="f32", seed=3, T=[0.0, 1.0])
    am = st.draft.float().argmax(dim=-1).to(torch.int32)
    for b in range(4):
        if float(st.temps[b]) == 0.0:
            assert torch.equal(st.tokens[b], am[b])


def test_sampled_tokens_follow_the_draft_softmax():
    # 20k draws from one row of softmax(z / T): chi-square against the law
    V, T, n = 6, 0.7, 20000
    z = torch.tensor([[[0.0, 1.0, -0.5, 2.0, 0.3, -2.0]]])
    g = torch.Generator().manual_seed(5)
    tok = workloads.sample_tokens(z, torch.tensor([T]), n, g)[0, :, 0].numpy()
    p = torch.softmax(z[0, 0] / T, dim=-1).numpy()
    obs = np.bincount(tok, minlength=V)
    chi2 = float(((obs - n * p) ** 2 / (n * p)).sum())
    assert chi2 < 20.5  # chi-square(5) at p = 0.001


def test_bf16_helpers_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10,
                        np.array([1.0, -0.0, 3.0078125, 3.01171875, 1e-30, 65504.0], np.float32)])
    bits = workloads.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    back = workloads.bf16_bits_to_f32(bits)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())
    # halfway cases go to the even neighbour
    half = np.array([0x3F808000, 0x3F818000], dtype=np.uint32).view(np.float32)
    assert list(workloads.f32_to_bf16_bits(half)) == [0x3F80, 0x3F82]


def test_host_inputs_are_the_same_bits():
    st = workloads.make_step(1, 3, B=2)
    tgt, drf, tok, tmp = workloads.host_inputs(st)
    assert tgt.dtype == np.uint16 and drf.dtype == np.uint16
    assert np.array_equal(workloads.bf16_bits_to_f32(tgt), st.target.float().numpy())
    assert np.array_equal(tok, st.tokens.numpy()) and np.array_equal(tmp, st.temps.numpy())


# -------------------------------------------------------- bench accounting
def _cfg(**kw):
    base = dict(index=9, name="t", B=4, gamma=3, V=1000, dtype="bf16", steps=1)
    base.update(kw)
    return workloads.Config(**base)


def test_step_bytes_closed_forms():
    cfg = _cfg()
    es, B, g, V = 2, 4, 3, 1000
    # the headline byte formula does not depend on temperatures or outcomes
    f = bench.step_bytes(cfg, torch.zeros(B))["formula"]
    assert f == B * (2 * g + 1) * V * es + B * V * es
    # all greedy: gamma + 1 target rows each, no draw
    assert bench.step_bytes(cfg, torch.zeros(B))["algorithmic"] == B * (g + 1) * V * es
    # all sampled, outcomes unknown: 2 gamma + 1 rows and one draw row each
    assert bench.step_bytes(cfg, torch.ones(B))["algorithmic"] == B * (2 * g + 2) * V * es
    # residual draws (accept_len < gamma) re-read two rows, the bonus draw
    # (accept_len = gamma) one, an invalid sequence (-1) none
    acc = torch.tensor([0, 2, 3, -1], dtype=torch.int32)
    got = bench.step_bytes(cfg, torch.ones(B), acc)["algorithmic"]
    assert got == ((2 * g + 1) * 4 + 2 + 2 + 1 + 0) * V * es
    # greedy rows ignore their accept length
    temps = torch.tensor([0.0, 1.0, 0.0, 1.0])
    got = bench.step_bytes(cfg, temps, torch.tensor([1, 1, 3, 3], dtype=torch.int32))["algorithmic"]
    assert got == (2 * (g + 1) + 2 * (2 * g + 1) + 2 + 1) * V * es
    # fp32 doubles every figure
    f32 = bench.step_bytes(_cfg(dtype="f32"), torch.ones(B))
    assert f32["algorithmic"] == 2 * bench.step_bytes(cfg, torch.ones(B))["algorithmic"]


def test_ring_exceeds_l2_or_is_capped():
    for cfg in workloads.CONFIGS:
        es = 2 if cfg.dtype == "bf16" else 4
        per = cfg.B * (2 * cfg.gamma + 1) * cfg.V * es
        r = bench.ring_size(cfg)
        assert r >= 8
        # at least 4x the L2 size of distinct inputs, unless that would pass ~24 GB
        assert r * per >= 4 * bench.L2_BYTES or r * per > 24e9 - per
        assert r * per <= max(24e9, 2 * per)


def test_clock_sampler_names_the_gpu_by_uuid(monkeypatch):
    """nvidia-smi counts physical GPUs and ignores CUDA_VISIBLE_DEVICES, so the
    sampler must name the device by its UUID, not by torch's index."""
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3")

    class Props:
        uuid = "5f0c2a4e-1111-2222-3333-444455556666"

    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda dev: Props())
    ident = bench.gpu_ident(0)
    assert ident == "GPU-5f0c2a4e-1111-2222-3333-444455556666"
    cmd = bench.ClockSampler(ident).command()
    assert cmd[:3] == ["nvidia-smi", "-i", ident]
    assert "0" not in cmd[1:3] and "3" not in cmd[1:3]


def test_rows_per_step():
    assert workloads.get(1).rows_per_step == 16 * 5
    assert workloads.get(3).rows_per_step == 8 * 4 * 5
    assert workloads.get(4).rows_per_step == 256 * 4


def test_clock_summary_from_sampled_rows(tmp_path):
    """The bench's clock record: median SM clock under load, the maximum,
    and every throttle reason seen active during the timed region."""
    rows = [
        "0, 1965, 1965, 300.5, 0x0, Not Active, Not Active, Not Active, Not Active, 0",
        "0, 1900, 1965, 610.0, 0x4, Not Active, Not Active, Not Active, Active, 98",
        "0, 1950, 1965, 640.2, 0x0, Not Active, Not Active, Not Active, Not Active, 100",
        "0, 1965, 1965, 655.9, 0x0, Not Active, Not Active, Not Active, Not Active, 100",
        "garbage line",
    ]
    p = tmp_path / "clk.csv"
    p.write_text("\n".join(rows) + "\n")
    c = bench.ClockSampler("GPU-x")
    c.path = str(p)
    s = c.summary()
    assert s["sm_mhz"] == 1950.0  # median of the three samples with load
    assert s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 655.9
    assert s["gpu"] == "GPU-x"
    c2 = bench.ClockSampler("GPU-x")
    c2.path = str(tmp_path / "missing.csv")
    assert c2.summary()["reasons"] == ["unavailable"]
