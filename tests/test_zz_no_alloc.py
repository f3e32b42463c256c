"""pa_decode_noalloc: decode attention for callers that cannot allocate device
memory (a runtime whose free memory all went to its KV-cache pool, plain C
hosts without a device allocator, loops that cannot take cudaMalloc's implicit
synchronisation).  Its split-K scratch is a fixed array inside the library, so
it is checked against pa_decode with a caller-provided workspace, through the
C ABI, on two calls in a row (the second call finds the first call's data in
the shared array): byte for byte, since both run the same kernels, and within
tolerance of the oracle.  Collected last so a failure here does not hide the
rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_443_b200 as pk
import workloads as W
from pa_harness import TOL, as_f64, build, oracle_attention, run_step

pytestmark = pytest.mark.gpu

LIMIT = 32 << 20


def _call_noalloc(out, p, spec, P):
    L = pk.lib()
    B, Hq, D = p.q.shape
    NB, Hkv, bs, _ = p.cache.k_cache.shape
    return L.pa_decode_noalloc(out.data_ptr(), p.q.data_ptr(), p.cache.k_cache.data_ptr(),
                               p.cache.v_cache.data_ptr(), p.tables.data_ptr(), p.tables.shape[1],
                               p.lens.data_ptr(), B, Hq, Hkv, D, bs, NB, spec.softmax_scale,
                               spec.dtype_code, P, p.max_ctx,
                               torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name,P", [("opt13b", 64), ("gqa70b", 128), ("tiny", 32)])
def test_noalloc_matches_workspace_decode_twice(name, P):
    """Both calls run the same kernels at the same partition length, so the
    output must be the same bytes as pa_decode's; it is also checked against
    the oracle.  The second call finds the first call's partials in the shared
    array, and must not depend on them."""
    pk.pa_device_status(clear=True)
    spec = W.small(name)
    p, o = build(W.scenario(spec))
    ref = run_step(p, spec, partition_size=P).clone()
    torch.cuda.synchronize()
    need = pk.pa_decode_workspace_bytes(p.q.shape[0], p.q.shape[1], spec.D, p.max_ctx, P)
    assert 0 < need <= LIMIT
    want = oracle_attention(o, spec)
    for _ in range(2):
        out = torch.full_like(p.q, float("nan"))
        assert _call_noalloc(out, p, spec, P) == pk.PA_OK, pk.pa_last_error()
        torch.cuda.synchronize()
        assert W.storage_view(out).tobytes() == W.storage_view(ref).tobytes()
        err = np.abs(as_f64(out, spec) - want).max()
        assert err <= TOL[spec.dtype], err
    assert pk.pa_device_status() == 0


def test_noalloc_rejects_batches_beyond_its_scratch():
    spec = W.small("opt13b")
    p, _ = build(W.scenario(spec), with_oracle=False)
    B, Hq, D = 4096, 64, 128               # needs ~1 GiB of partials at 32-token partitions
    assert pk.pa_decode_workspace_bytes(B, Hq, D, 1024, 32) > LIMIT
    n0 = pk.pa_launch_count()
    L = pk.lib()
    st = L.pa_decode_noalloc(p.q.data_ptr(), p.q.data_ptr(), p.cache.k_cache.data_ptr(),
                             p.cache.v_cache.data_ptr(), p.tables.data_ptr(), 64,
                             p.lens.data_ptr(), B, Hq, 8, D, 16, p.cache.num_blocks, 0.1,
                             spec.dtype_code, 32, 1024, None)
    assert st == pk.PA_ERR_UNSUPPORTED
    assert "scratch" in pk.pa_last_error()
    assert pk.pa_launch_count() == n0
