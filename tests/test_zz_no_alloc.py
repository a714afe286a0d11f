"""The decode entry point that allocates nothing (pkv_paged_attention_decode_noalloc).

It serves callers that cannot allocate device memory, such as code inside a
host runtime that owns every device allocation and offers its plugins no
allocator or workspace.  Its split-K scratch is a fixed 16 MiB device array
inside the library, shared by every call.  These tests call it through the
C ABI and check its output against pkv_paged_attention_decode (which takes a
caller-allocated workspace) with the tolerances the parity tests use, on two
calls in a row (the second call finds the first call's leftovers in the
shared scratch).  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_439_b200.workloads import make_custom

from pkv_testlib import GpuCache, OracleCache, assert_close, tol_for

pytestmark = pytest.mark.gpu


def _cases():
    return [
        # long, uneven contexts on few (sequence, kv head) units: many splits
        make_custom("noalloc-gqa8-bf16", [3000, 4097, 17, 1500], 16, 2, 128, 16, "bf16", seed=21),
        make_custom("noalloc-mha-int8", [700, 2049, 33], 4, 4, 128, 16, "i8", seed=22,
                    outlier_prob=0.01),
        make_custom("noalloc-gqa4-bs256", [5000, 260, 999], 8, 2, 64, 256, "bf16", seed=23),
        make_custom("noalloc-gqa2-fp8", [1800, 2600, 90], 4, 2, 128, 16, "fp8", seed=24,
                    outlier_prob=0.01),
    ]


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
@pytest.mark.parametrize("splits", [0, 5])
def test_noalloc_matches_workspace_entry_point(idx, splits):
    import paged_kv_cache_439_b200 as pkv
    wl = _cases()[idx]
    g = GpuCache(wl).fill()
    dev = g.device
    q, bt, cl = wl.q.to(dev), wl.block_tables.to(dev), wl.context_lens.to(dev)
    common = dict(softmax_scale=wl.softmax_scale, k_scale=g.ks, v_scale=g.vs,
                  max_context_len=wl.max_context_len, num_splits=splits, err_flag=g.err)
    need = pkv.workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                              wl.max_context_len, g.k.dtype, splits)
    assert 0 < need <= 16 * 1024 * 1024   # split-K is in use and fits the fixed scratch
    ref = pkv.paged_attention_decode(q, g.k, g.v, bt, cl, **common)
    tol = tol_for(wl)
    outs = []
    for _ in range(2):                    # two calls in a row share the scratch
        out = torch.full_like(q, float("nan"))
        pkv.paged_attention_decode_noalloc(q, g.k, g.v, bt, cl, out=out, **common)
        outs.append(out)
    torch.cuda.synchronize()
    ref_np = ref.float().cpu().numpy().astype(np.float64)
    for out in outs:
        assert_close(out, ref_np, tol, f"{wl.name} splits={splits}")
    assert g.flags() == 0
    # and both agree with the oracle
    oracle_out = OracleCache(wl).fill().decode()
    for out in outs:
        assert_close(out, oracle_out, tol, f"{wl.name} vs oracle")


def test_noalloc_rejects_shapes_beyond_the_scratch():
    from paged_kv_cache_439_b200 import _native as N
    lib = N.lib()
    B, nq, nkv, d, maxctx, splits = 256, 64, 8, 128, 32768, 16
    need = lib.pkv_workspace_size(B, nq, nkv, d, maxctx, N.PKV_BF16, splits)
    assert need > N.NOALLOC_SCRATCH_BYTES
    # rejected before any launch: these buffers are never touched
    t = torch.empty(64, dtype=torch.uint8, device="cuda")
    p = t.data_ptr()
    rc = lib.pkv_paged_attention_decode_noalloc(
        p, p, N.PKV_BF16, p, p, N.PKV_BF16, None, None, p, maxctx // 16, p, maxctx, B, nq, nkv, d,
        16, 4096, 0.1, splits, None, None)
    assert rc == N.PKV_ERR_SCRATCH_LIMIT
    assert b"no-allocation" in lib.pkv_strerror(rc)
