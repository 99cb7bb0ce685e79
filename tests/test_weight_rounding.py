"""How far the rounding of the softmax weights P to a 16-bit type can move an
attention output, on the CPU.

The bf16 tcgen05 kernels compute E_j = exp2(s_j - m) in fp32 (the row's
largest weight is exp2(0) = 1, exact), round each E_j to f16 for the P V
product and divide by l = sum_j E_j taken in fp32 from the unrounded weights.
The output therefore moves by sum_j (P_j - E_j) V_j / l.  Round to nearest
moves each weight by at most u E_j (u = 2^-11 for f16's 11 significant bits,
2^-8 for bf16's 8), except below f16's normal range (E_j < 2^-14), where the
subnormal spacing 2^-24 allows up to 2^-25 whatever E_j.  So the output moves
by at most u times the attention-weighted mean of |V| (at most u max|V|) plus,
in f16, 2^-25 sum_{E_j < 2^-14} |V_j| / l.  These tests check that bound on
random rows, and that rows built for each term (weights just above a power
of two, or just under half the subnormal spacing, each error with the sign of
its V) come within 1 % of it: the first term is u max|V|, not u/2 max|V|.
"""

import numpy as np
import pytest
import torch

U = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}
# below this a weight is subnormal in the type, and rounds by up to SUB_ERR
SUB_MIN = {torch.float16: 2.0 ** -14, torch.bfloat16: 2.0 ** -126}
SUB_ERR = {torch.float16: 2.0 ** -25, torch.bfloat16: 2.0 ** -134}


def bound(logits2, v, dtype):
    """u * sum_{normal} E|V| / l + sub_err * sum_{subnormal} |V| / l per row."""
    e = np.exp2(logits2 - logits2.max(axis=-1, keepdims=True)).astype(np.float32).astype(np.float64)
    normal = e >= SUB_MIN[dtype]
    l = e.sum(axis=-1)
    return (U[dtype] * (np.where(normal, e, 0.0) * np.abs(v)).sum(axis=-1)
            + SUB_ERR[dtype] * (np.where(normal, 0.0, 1.0) * np.abs(v)).sum(axis=-1)) / l


def weight_rounding_shift(logits2: np.ndarray, v: np.ndarray, dtype) -> np.ndarray:
    """Per row: sum_j (round(E_j) - E_j) v_j / sum_j E_j with E = exp2(s - max s)
    in fp32, rounded to `dtype` by a round-to-nearest cast, the shift in fp64."""
    e = np.exp2(logits2 - logits2.max(axis=-1, keepdims=True)).astype(np.float32)
    p = torch.from_numpy(e).to(dtype).to(torch.float64).numpy()
    e64 = e.astype(np.float64)
    return ((p - e64) * v).sum(axis=-1) / e64.sum(axis=-1)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_bound_holds_on_random_rows(dtype):
    rng = np.random.default_rng(0)
    u = U[dtype]
    for n, temp in [(2, 1.0), (16, 0.3), (128, 3.0), (1024, 1.0), (1024, 8.0), (4096, 0.05)]:
        s = rng.standard_normal((256, n)) * temp * 8.0
        v = rng.standard_normal((256, n)) * 3.0
        shift = weight_rounding_shift(s, v, dtype)
        # the exact weights are the fp32 ones; fp64 sums add ~1e-16 relative
        assert np.all(np.abs(shift) <= bound(s, v, dtype) * (1 + 1e-6) + 1e-15), (n, temp)
        if temp < 1.0:  # no weight of these rows is subnormal in either type
            assert np.all(np.abs(shift) <= u * np.abs(v).max(axis=-1) * (1 + 1e-6) + 1e-15)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_bound_is_reached(dtype):
    """One weight of 1 (exact) and n - 1 weights just above 1/2, each rounded
    down by almost half an ulp, with v = -M: the shift approaches u M."""
    u = U[dtype]
    n, big_v = 4096, 9.0
    half_ulp = u / 2  # half an ulp of the binade [1/2, 1)
    w = 0.5 + half_ulp * (1 - 2.0 ** -12)  # rounds down to 1/2, error just under half an ulp
    logits2 = np.full((1, n), np.log2(w))
    logits2[0, 0] = 0.0
    e = np.exp2(logits2 - logits2.max()).astype(np.float32)
    assert e[0, 0] == 1.0 and abs(float(e[0, 1]) - w) < 2.0 ** -20  # fp32 exp2 lands where intended
    v = np.full((1, n), -big_v)
    v[0, 0] = 0.0
    shift = float(weight_rounding_shift(logits2, v, dtype)[0])
    assert shift > 0.0
    assert shift <= u * big_v
    assert shift >= 0.99 * u * big_v
    assert shift > 1.9 * (u / 2) * big_v  # twice what half the unit roundoff would allow


def test_f16_weights_and_the_flat_gate():
    """The flat 2e-2 gate below |O| = 8: the output's own rounding (half a bf16
    ulp, 2^-6 in [4, 8)) plus the f16 weights' worst case u max|V| stays under
    2e-2 exactly when max|V| < (2e-2 - 2^-6) 2^11 = 8.96; with bf16 weights it
    does not even at max|V| = 1.2."""
    out_half_ulp = 2.0 ** -6
    assert out_half_ulp + U[torch.float16] * 8.95 < 2e-2 < out_half_ulp + U[torch.float16] * 8.97
    # the workloads' largest |V|: 8.8125 (128K, block-sparse) under it, 9.125 (32K) over it
    assert out_half_ulp + U[torch.float16] * 8.8125 < 2e-2 < out_half_ulp + U[torch.float16] * 9.125
    assert out_half_ulp + U[torch.bfloat16] * 1.2 > 2e-2


def test_subnormal_weights_term_is_reached():
    """One weight of 1 and n - 1 f16-subnormal weights just under half the
    subnormal spacing (each rounds to 0, an error of almost 2^-25), v = -M:
    the shift approaches 2^-25 (n - 1) M / l, the bound's second term, which
    u E |V| alone would put 2^14 times lower."""
    n, big_v = 4096, 9.0
    w = 2.0 ** -25 * (1 - 2.0 ** -10)
    logits2 = np.full((1, n), np.log2(w))
    logits2[0, 0] = 0.0
    v = np.full((1, n), -big_v)
    v[0, 0] = 0.0
    shift = float(weight_rounding_shift(logits2, v, torch.float16)[0])
    b = float(bound(logits2, v, torch.float16)[0])
    assert 0.99 * b <= shift <= b
    assert shift > 1000 * U[torch.float16] * w * (n - 1) * big_v
    # bf16 has the fp32 exponent range: the same row is rounded almost exactly
    assert abs(float(weight_rounding_shift(logits2, v, torch.bfloat16)[0])) <= U[torch.bfloat16] * w * (n - 1) * big_v
