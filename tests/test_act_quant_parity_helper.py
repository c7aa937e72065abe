"""The parity check of the activation-quantized modes (helpers.
assert_parity_act_quant), on the CPU: a simulated GPU result whose h codes
differ from the oracle's only where fp32 rounding leaves them undetermined
must pass, and results with real errors must fail.  No GPU."""
import numpy as np
import pytest

import oracle
from block_quantized_expert_mxfp4_b200 import synth
from helpers import _quant_at, act_quant_alternatives, assert_parity, assert_parity_act_quant
from ref_decode import dequant_mx

E, H, I, T, K = 6, 1024, 512, 4, 3


def _setup(seed=0):
    rng = np.random.default_rng(seed)
    ws = []
    for rows, cols in ((I, H), (I, H), (H, I)):
        ws.append((rng.integers(0, 256, (E, rows, cols // 2), dtype=np.uint8),
                   rng.integers(118, 128, (E, rows, cols // 32), dtype=np.uint8)))
    L = oracle.Layer(*[oracle.Weight(oracle.MXFP4, q, s) for q, s in ws])
    x = synth.activations(seed, T, H)
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    w = rng.dirichlet(np.ones(K), T)
    return ws, L, x, ids, w


def _simulate(ws, L, x, ids, w, aq, mutate):
    """y from the oracle's g, u with h handled by `mutate(h32, hq) -> hq'`,
    down in fp64, output rounded to fp32 (the GPU's y)."""
    y = np.zeros((T, H))
    for t in range(T):
        for s in range(K):
            e = ids[t, s]
            g, u, hq, _ = oracle.expert_ffn(L, e, x[t], aq)
            h32 = (g / (1.0 + np.exp(-g)) * u).astype(np.float32).astype(np.float64)
            y[t] += w[t, s] * (dequant_mx(*[a[e] for a in ws[2]]) @ mutate(h32, hq))
    return y.astype(np.float32)


@pytest.mark.parametrize("aq", [oracle.ACT_MXFP4, oracle.ACT_E4M3])
def test_undetermined_codes_taken_the_other_way_pass(aq):
    ws, L, x, ids, w = _setup(1)
    flipped = [0]

    def flip_all(h32, hq):
        out = hq.copy()
        for idx, alt in act_quant_alternatives(h32, hq, aq, 2.0 ** -13):
            if idx.size == 1:
                out[idx] = alt
                flipped[0] += 1
        return out

    y = _simulate(ws, L, x, ids, w, aq, flip_all)
    assert flipped[0] > 0
    e, c, used, offered = assert_parity_act_quant(y, L, x, ids, w, aq)
    assert used >= 1 and offered >= flipped[0]


def test_flips_matter_for_the_plain_bar():
    """Without the alternatives the same simulated result can miss the bar:
    the reason the check exists (e2m1 steps are a third of a value or more)."""
    ws, L, x, ids, w = _setup(1)
    aq = oracle.ACT_MXFP4

    def flip_all(h32, hq):
        out = hq.copy()
        for idx, alt in act_quant_alternatives(h32, hq, aq, 2.0 ** -9):
            if idx.size == 1:
                out[idx] = alt
        return out

    y = _simulate(ws, L, x, ids, w, aq, flip_all)
    with pytest.raises(AssertionError):
        assert_parity(y, oracle.moe_forward(L, x, ids, w, aq))


@pytest.mark.parametrize("aq", [oracle.ACT_MXFP4, oracle.ACT_E4M3])
@pytest.mark.parametrize("bug", ["h_unquantized", "scale_off_by_one", "x_unquantized_h_from_plain"])
def test_real_errors_fail(aq, bug):
    ws, L, x, ids, w = _setup(2)
    emax = 2 if aq == oracle.ACT_MXFP4 else 8
    if bug == "h_unquantized":
        y = _simulate(ws, L, x, ids, w, aq, lambda h32, hq: h32)
    elif bug == "scale_off_by_one":
        def wrong_scale(h32, hq):  # every block one binade coarser than the rule
            out = np.empty_like(hq)
            for b in range(h32.size // 32):
                v = h32[32 * b:32 * b + 32]
                _, ex = np.frexp(np.abs(v).max())
                out[32 * b:32 * b + 32] = _quant_at(v, ex - 1 - emax + 1, aq)
            return out
        y = _simulate(ws, L, x, ids, w, aq, wrong_scale)
    else:
        y = oracle.moe_forward(L, x, ids, w).astype(np.float32)  # the bf16 path's result
    with pytest.raises(AssertionError):
        assert_parity_act_quant(y, L, x, ids, w, aq)
