"""The bf16 output check of the parity tests can fail (CPU; no GPU needed).

On the benchmark workloads the logits have a standard deviation of about 0.25,
so attention is near-uniform over thousands of keys and each output element is
about 1e-2 in size.  An absolute bound of 2e-2 alone would then pass a PV
product that lost a whole 128-key V tile.  Here mistakes of that kind are
planted in the float64 oracle's inputs, at the shape of one (chunk, KV head)
group of the 2048-slot / 1024-token workload, and the checker must reject each
of them while it accepts outputs that carry only the rounding a correct bf16
kernel makes (P rounded to bf16 before the PV product, fp32 accumulation, the
output rounded to bf16).
"""
import math

import numpy as np
import pytest
import torch

from oracle import attend_group
from tests.parity_util import OUT_RELNORM_BF16, check_outputs

G, S, NV, D = 4, 1024, 2048, 128


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


@pytest.fixture(scope="module")
def group():
    rng = np.random.default_rng(5)
    q = _bf16(rng.standard_normal((G, S, D)) * 0.5)
    kc, vc = (_bf16(rng.standard_normal((NV, D)) * 0.5) for _ in range(2))
    kn, vn = (_bf16(rng.standard_normal((S, D)) * 0.5) for _ in range(2))
    valid = np.ones(NV, bool)
    ref, _, _ = attend_group(q, kc, vc, valid, kn, vn, 1.0 / math.sqrt(D))
    return q, kc, vc, kn, vn, valid, ref


def _bf16_kernel_like(q, kc, vc, kn, vn):
    """Outputs as a correct bf16 kernel forms them: exact p rounded to bf16,
    the PV product accumulated in float32, the result rounded to bf16."""
    keys = np.concatenate([kc, kn])
    vals = np.concatenate([vc, vn]).astype(np.float32)
    out = np.empty((G, S, D))
    for g in range(G):
        s = q[g] @ keys.T / math.sqrt(D)
        s[:, NV:][np.arange(S)[None, :] > np.arange(S)[:, None]] = -np.inf
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        out[g] = _bf16(_bf16(p).astype(np.float32) @ vals)
    return out


def test_bf16_rounding_alone_passes(group):
    q, kc, vc, kn, vn, _, ref = group
    r = check_outputs(_bf16_kernel_like(q, kc, vc, kn, vn), ref, torch.bfloat16, "rounding only")
    # the reading recorded with the tolerances: rounding gives a few 1e-3
    assert r["rel_norm"] < 0.5 * OUT_RELNORM_BF16, r


@pytest.mark.parametrize("slip", ["drop-cache-tile", "drop-chunk-tile", "swap-tiles", "shift-head"])
def test_planted_pv_slips_fail(group, slip):
    q, kc, vc, kn, vn, valid, ref = group
    vc2, vn2 = vc.copy(), vn.copy()
    scale = 1.0 / math.sqrt(D)
    if slip == "drop-cache-tile":          # one 128-key V tile of the cache never added
        vc2[1024:1152] = 0.0
        bad, _, _ = attend_group(q, kc, vc2, valid, kn, vn, scale)
    elif slip == "drop-chunk-tile":        # the chunk's last V tile lost
        vn2[896:] = 0.0
        bad, _, _ = attend_group(q, kc, vc, valid, kn, vn2, scale)
    elif slip == "swap-tiles":             # two V tiles read from each other's rows
        vc2[0:128], vc2[128:256] = vc[128:256], vc[0:128]
        bad, _, _ = attend_group(q, kc, vc2, valid, kn, vn, scale)
    else:                                  # head g's output written as head g + 1's
        bad = np.roll(ref, 1, axis=0)
    # max |delta| stays inside the absolute bound for the tile slips: only the
    # relative norm catches them
    with pytest.raises(AssertionError):
        check_outputs(_bf16(bad), ref, torch.bfloat16, slip)
