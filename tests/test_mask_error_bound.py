"""The tensor-core mask build's logit error bound, against emulations of its arithmetic (CPU).

The build stores each exact block mean x as three bf16 pieces b1 + b2 + b3 (each the rounded
remainder of the previous ones, from the float32 value of x) plus a float32 residual, and takes
the fast pooled logit as s = (D1 + D2) * scale with D1 = b1.b1 and D2 = b1.b2 + b2.b1 + b1.b3 +
b2.b2 + b3.b1, accumulated in fp32 on the tensor cores.  Rows whose order near the CDF boundary
could differ from the float64 order by more than E = 2^-15 * scale * |Qp_i| * max_j |Kp_j| are
recomputed in float64, so the mask is exact only if |s - s_exact| < E always holds.

The tensor core's internal summation of a 16-product step is not documented; two models are
emulated here: (a) every product added to the fp32 accumulator with round to nearest, one at a
time; (b) each step's 16 products aligned to the largest and cut to 24 bits below it (truncation),
then added to the accumulator.  Inputs: block means of the seeded synthetic q and k (the shapes
and distributions the GPU tests use) and adversarial means with heavy cancellation.
"""
import numpy as np
import pytest

import dbst_synth as S

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16(x):
    """Round float32 values to bf16 (round to nearest even), returned as float64."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def pieces(x):
    hi = f32(x)
    b1 = bf16(hi)
    r1 = f32(hi - b1)
    b2 = bf16(r1)
    r2 = f32(r1 - b2)
    b3 = bf16(r2)
    res = f32(x - (b1 + b2 + b3))
    return b1, b2, b3, res


def acc_rn(prods):
    """Model (a): fp32 accumulation, one product at a time, round to nearest."""
    acc = np.zeros(prods.shape[:-1], dtype=np.float32)
    for c in range(prods.shape[-1]):
        acc = (acc + prods[..., c].astype(np.float32)).astype(np.float32)
    return acc.astype(np.float64)


def acc_trunc(prods, k=16):
    """Model (b): steps of k products aligned to the largest and truncated to 24 bits below it."""
    acc = np.zeros(prods.shape[:-1], dtype=np.float32)
    for s0 in range(0, prods.shape[-1], k):
        step = prods[..., s0:s0 + k]
        m = np.max(np.abs(step), axis=-1, keepdims=True)
        e = np.floor(np.log2(np.where(m > 0, m, 1.0)))
        ulp = np.exp2(e - 23)
        t = np.trunc(step / ulp) * ulp                 # toward zero, on the largest product's grid
        acc = (acc + t.sum(-1).astype(np.float32)).astype(np.float32)
    return acc.astype(np.float64)


def check(qp, kp, scale):
    q1, q2, q3, _ = pieces(qp)
    k1, k2, k3, _ = pieces(kp)
    exact = qp @ kp.T * scale
    E = 2.0 ** -15 * scale * np.linalg.norm(qp, axis=1)[:, None] * np.linalg.norm(kp, axis=1).max() * 1.001
    worst = 0.0
    for acc in (acc_rn, acc_trunc):
        d1 = acc(q1[:, None, :] * k1[None, :, :])
        cross = (q1[:, None, :] * k2[None] + q2[:, None, :] * k1[None] + q1[:, None, :] * k3[None] +
                 q2[:, None, :] * k2[None] + q3[:, None, :] * k1[None])
        d2 = acc(cross)
        fast = f32(f32(d1 + d2) * f32(scale))
        worst = max(worst, float(np.max(np.abs(fast - exact) / E)))
    return worst


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_bound_holds_on_the_synthetic_block_means(name):
    w = S.workload(name)
    q, k, _ = S.make_qkv(w)
    # block means of 64 consecutive raster tokens per head (the tiling does not matter for the bound)
    to64 = lambda a: S.f32_from_bf16_bits(a).astype(np.float64)   # noqa: E731
    qm = to64(q)[0, 0].reshape(-1, 64, w.D).mean(1)
    km = to64(k)[0, 0].reshape(-1, 64, w.D).mean(1)
    worst = check(qm, km, 1.0 / np.sqrt(w.D))
    assert worst < 1.0, worst
    assert worst < 0.25   # the bound's margin is not used up


def test_bound_holds_under_cancellation():
    rng = np.random.default_rng(5)
    D = 128
    base = rng.normal(size=(D,))
    # logits that cancel to small values: keys nearly orthogonal to the queries, large entries
    qp = np.stack([base * 10.0 + rng.normal(size=D) * 1e-3 for _ in range(16)])
    kp = rng.normal(size=(64, D)) * 10.0
    kp -= np.outer(kp @ base / (base @ base), base)      # orthogonal to base
    kp += rng.normal(size=(64, D)) * 1e-4
    worst = check(qp, kp, 1.0 / np.sqrt(D))
    assert worst < 1.0, worst
