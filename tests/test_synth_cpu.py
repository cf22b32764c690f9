"""The seeded synthetic inputs follow their stated recipe (kda_synth's docstring): unit q/k rows,
the two decay distributions, beta in (0, 1), the initial-state scale, log-uniform varlen lengths
inside their bounds, and reproducibility from the seed."""
import math

import numpy as np
import pytest
import torch

import kda_synth
from kda_synth import PrefillSpec


def _spec(dtype="f32", decay="fast", init_std=0.02, **kw):
    args = dict(B=2, T=512, H=4, Dk=32, Dv=16, chunk=64)
    args.update(kw)
    return PrefillSpec("t", dtype=dtype, decay=decay, init_std=init_std, **args)


def _softplus_mean(shift, n=400_000, seed=5):
    z = np.random.Generator(np.random.PCG64(seed)).standard_normal(n) + shift
    return float(np.mean(np.logaddexp(0.0, z)))


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 1e-2)])
def test_query_and_key_rows_have_unit_norm(dtype, tol):
    x = kda_synth.prefill_inputs(_spec(dtype=dtype), 3)
    for n in ("q", "k"):
        norms = x[n].double().norm(dim=-1)
        assert torch.all((norms - 1).abs() <= tol), n
    assert x["q"].dtype == kda_synth.torch_dtype(dtype) and x["log_alpha"].dtype == torch.float32


@pytest.mark.parametrize("decay,scale,shift", [("fast", 0.5, 0.0), ("slow", 1.0, -2.0)])
def test_decay_distributions(decay, scale, shift):
    x = kda_synth.prefill_inputs(_spec(decay=decay, T=4096), 4)
    la = x["log_alpha"].double()
    assert torch.all(la < 0) and torch.isfinite(la).all()
    # mean of -scale * softplus(N(shift, 1)), against a numpy Monte Carlo of the same formula
    assert float(la.mean()) == pytest.approx(-scale * _softplus_mean(shift), rel=0.02)


def test_beta_values_and_initial_state_scale():
    x = kda_synth.prefill_inputs(_spec(T=4096), 6)
    b = x["beta"]
    assert torch.all((b > 0) & (b < 1)) and float(b.mean()) == pytest.approx(0.5, abs=0.01)
    assert tuple(x["initial_state"].shape) == (2, 4, 32, 16)
    assert float(x["initial_state"].std()) == pytest.approx(0.02, rel=0.05)
    assert float(x["v"].std()) == pytest.approx(1.0, rel=0.02)
    assert kda_synth.prefill_inputs(_spec(init_std=0.0), 6)["initial_state"] is None


def test_varlen_lengths_and_offsets():
    lens = kda_synth.loguniform_lengths(2000, 256, 32768, 11)
    assert min(lens) >= 256 and max(lens) <= 32768
    # log-uniform: the median sits near the geometric mean of the bounds
    assert np.median(lens) == pytest.approx(math.sqrt(256 * 32768), rel=0.15)
    assert lens == kda_synth.loguniform_lengths(2000, 256, 32768, 11)
    spec = kda_synth.varlen_spec(1003, n=6, lo=16, hi=512)
    assert list(spec.seqlens) == kda_synth.loguniform_lengths(6, 16, 512, 1003)
    x = kda_synth.prefill_inputs(spec, 1, "cpu")
    cu = x["cu_seqlens"].long().numpy()
    assert cu[0] == 0 and list(np.diff(cu)) == list(spec.seqlens)
    assert x["q"].shape[:2] == (1, spec.total_tokens)
    with pytest.raises(ValueError):
        kda_synth.prefill_inputs(PrefillSpec("v", B=2, T=10, H=1, Dk=8, Dv=8, chunk=16,
                                             dtype="f32", decay="fast", init_std=0.0,
                                             seqlens=(4, 6)), 1)


def test_inputs_are_reproducible_from_the_seed():
    a = kda_synth.prefill_inputs(_spec(), 21)
    b = kda_synth.prefill_inputs(_spec(), 21)
    c = kda_synth.prefill_inputs(_spec(), 22)
    for n in ("q", "k", "v", "log_alpha", "beta", "initial_state"):
        assert torch.equal(a[n], b[n]), n
        assert not torch.equal(a[n], c[n]), n


def test_decode_steps_share_their_prefix():
    spec = kda_synth.DecodeSpec("d", N=3, H=2, Dk=16, Dv=8, steps=5, dtype="f32", decay="slow",
                                init_std=0.02)
    long = kda_synth.decode_step_inputs(spec, 30, 5)
    short = kda_synth.decode_step_inputs(spec, 30, 3)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        assert torch.equal(long[n][:3], short[n]), n
    assert tuple(kda_synth.decode_state(spec, 30).shape) == (3, 2, 16, 8)
