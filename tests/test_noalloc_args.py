"""The binding of h2o_attend_noalloc rejects bad buffers before any pointer
reaches the library (CPU; no call here reaches the C ABI).

The library reads and writes through raw pointers: a cache with fewer than M
rows, a non-contiguous or wrongly typed buffer, or an output too small would
make its kernels read or write past the buffers, so each case must raise
ValueError in Python first.
"""
import pytest
import torch

import h2o_kv_cache_b200 as h2o

B, Hq, Hkv, S, D, M = 1, 4, 2, 8, 64, 32


def _bufs(dtype=torch.float32):
    q = torch.zeros(B, Hq, S, D, dtype=dtype)
    k = torch.zeros(B, Hkv, S, D, dtype=dtype)
    v = torch.zeros(B, Hkv, S, D, dtype=dtype)
    kc = torch.zeros(B, Hkv, M, D, dtype=dtype)
    vc = torch.zeros(B, Hkv, M, D, dtype=dtype)
    out = torch.zeros(B, Hq, S, D, dtype=dtype)
    cs = torch.zeros(B, Hkv, M + S, dtype=torch.float32)
    return dict(q=q, k=k, v=v, k_cache=kc, v_cache=vc, out=out, colsum=cs)


def _call(n_valid=16, **over):
    a = _bufs()
    a.update(over)
    return h2o.attend_noalloc(a["q"], a["k"], a["v"], a["k_cache"], a["v_cache"], n_valid=n_valid,
                              M=M, out=a["out"], colsum=a["colsum"])


@pytest.mark.parametrize("case,over,n_valid,msg", [
    ("q dtype", dict(q=torch.zeros(B, Hq, S, D, dtype=torch.float16)), 16, "float32 or bfloat16"),
    ("q rank", dict(q=torch.zeros(Hq, S, D)), 16, "4-d"),
    ("k dtype", dict(k=torch.zeros(B, Hkv, S, D, dtype=torch.bfloat16)), 16, "k must be"),
    ("k heads", dict(k=torch.zeros(B, 3, S, D), v=torch.zeros(B, 3, S, D)), 16, "multiple of Hkv"),
    ("v shape", dict(v=torch.zeros(B, Hkv, S + 1, D)), 16, "v must have shape"),
    ("k not contiguous", dict(k=torch.zeros(B, Hkv, D, S).transpose(2, 3)), 16, "contiguous"),
    ("short cache", dict(k_cache=torch.zeros(B, Hkv, M - 1, D)), 16, "k_cache must have shape"),
    ("cache dtype", dict(v_cache=torch.zeros(B, Hkv, M, D, dtype=torch.bfloat16)), 16, "v_cache must be"),
    ("missing cache", dict(k_cache=None), 16, "required"),
    ("n_valid > M", {}, M + 1, "n_valid"),
    ("n_valid < 0", {}, -1, "n_valid"),
    ("small out", dict(out=torch.zeros(B, Hq, S - 1, D)), 16, "out must have shape"),
    ("out dtype", dict(out=torch.zeros(B, Hq, S, D, dtype=torch.bfloat16)), 16, "out must be"),
    ("colsum dtype", dict(colsum=torch.zeros(B, Hkv, M + S, dtype=torch.float64)), 16, "colsum must be"),
    ("short colsum", dict(colsum=torch.zeros(B, Hkv, M)), 16, "colsum must have shape"),
    ("colsum not contiguous", dict(colsum=torch.zeros(B, M + S, Hkv).transpose(1, 2)), 16, "contiguous"),
])
def test_rejects_bad_buffers(case, over, n_valid, msg):
    with pytest.raises(ValueError, match=msg):
        _call(n_valid=n_valid, **over)


def test_rejects_host_tensors_last():
    # well-formed buffers that are not CUDA tensors never reach the library either
    with pytest.raises(ValueError, match="CUDA tensor"):
        _call()
    # an empty cache may be passed as None
    with pytest.raises(ValueError, match="CUDA tensor"):
        _call(n_valid=0, k_cache=None, v_cache=None)
