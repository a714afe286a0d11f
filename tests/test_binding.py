"""Host-side checks of the Python binding (no GPU needed).

The C ABI receives raw pointers plus sizes, so it cannot see a tensor that is
smaller than the sizes passed with it.  The binding derives those sizes from
the tensors and refuses inconsistent ones before anything reaches the library;
these tests drive each refusal with CPU tensors (the shape checks run before
the device checks), then check that consistent CPU tensors are refused for
not being on a CUDA device."""
import pytest
import torch

import paged_kv_cache_439_b200 as pkv

B, NQ, NKV, D, NB, BS = 3, 8, 2, 64, 12, 16


def _decode_args(cache_dtype=torch.bfloat16):
    q = torch.zeros(B, NQ, D, dtype=torch.bfloat16)
    kc = torch.zeros(NB, BS, NKV, D, dtype=torch.bfloat16).to(cache_dtype)
    vc = kc.clone()
    bt = torch.zeros(B, 4, dtype=torch.int32)
    cl = torch.ones(B, dtype=torch.int32)
    return q, kc, vc, bt, cl


def _scales():
    return (torch.ones(NB, NKV, BS, dtype=torch.float32),
            torch.ones(NB, NKV, BS, dtype=torch.float32))


def test_consistent_cpu_tensors_are_refused_for_their_device():
    q, kc, vc, bt, cl = _decode_args()
    with pytest.raises(ValueError, match="CUDA"):
        pkv.paged_attention_decode(q, kc, vc, bt, cl, workspace=torch.empty(16, dtype=torch.uint8))
    k = torch.zeros(B, NKV, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        pkv.kv_cache_append(k, k.clone(), torch.zeros(B, dtype=torch.int64), kc, vc)


def test_cache_shapes_must_agree():
    q, kc, vc, bt, cl = _decode_args()
    with pytest.raises(ValueError, match="k_cache and v_cache"):
        pkv.paged_attention_decode(q, kc, vc[:-1], bt, cl)
    with pytest.raises(ValueError, match="head_dim"):
        pkv.paged_attention_decode(torch.zeros(B, NQ, 128, dtype=torch.bfloat16), kc, vc, bt, cl)
    with pytest.raises(ValueError, match="k_cache and v_cache"):
        pkv.paged_attention_decode(q, kc[0], vc[0], bt, cl)


def test_scales_must_cover_the_pool():
    q, kc, vc, bt, cl = _decode_args(torch.int8)
    ks, vs = _scales()
    with pytest.raises(ValueError, match="k_scale and v_scale"):
        pkv.paged_attention_decode(q, kc, vc, bt, cl, k_scale=ks[:-1], v_scale=vs)
    with pytest.raises(ValueError, match="k_scale and v_scale"):
        pkv.paged_attention_decode(q, kc, vc, bt, cl, k_scale=ks, v_scale=vs.double())


def test_tables_must_cover_every_sequence():
    q, kc, vc, bt, cl = _decode_args()
    with pytest.raises(ValueError, match="block_tables"):
        pkv.paged_attention_decode(q, kc, vc, bt[:-1], cl)
    with pytest.raises(ValueError, match="block_tables"):
        pkv.paged_attention_decode(q, kc, vc, bt, cl[:-1])
    with pytest.raises(TypeError, match="int32"):
        pkv.paged_attention_decode(q, kc, vc, bt.long(), cl)


def test_out_and_err_flag_must_fit():
    q, kc, vc, bt, cl = _decode_args()
    with pytest.raises(ValueError, match="out"):
        pkv.paged_attention_decode(q, kc, vc, bt, cl, out=q[:-1].clone())
    with pytest.raises(ValueError, match="out"):
        pkv.paged_attention_decode(q, kc, vc, bt, cl, out=q.float())
    with pytest.raises(ValueError, match="err_flag"):
        pkv.paged_attention_decode(q, kc, vc, bt, cl, err_flag=torch.zeros(1, dtype=torch.int64))


def test_new_tokens_must_match_the_batch_and_cache():
    q, kc, vc, bt, cl = _decode_args()
    k = torch.zeros(B, NKV, D, dtype=torch.bfloat16)
    slots = torch.zeros(B, dtype=torch.int64)
    with pytest.raises(ValueError, match="num_tokens"):
        pkv.paged_attention_decode_append(q, k[:-1], k[:-1].clone(), slots, kc, vc, bt, cl)
    with pytest.raises(ValueError, match="num_tokens"):
        pkv.paged_attention_decode_append(q, k, k.clone(), slots[:-1], kc, vc, bt, cl)
    with pytest.raises(TypeError, match="int64"):
        pkv.paged_attention_decode_append(q, k, k.clone(), slots.int(), kc, vc, bt, cl)
    with pytest.raises(ValueError, match="q's dtype"):
        pkv.paged_attention_decode_append(q, k.float(), k.float(), slots, kc, vc, bt, cl)
    with pytest.raises(ValueError, match="kv heads"):
        pkv.kv_cache_append(torch.zeros(B, NKV + 1, D, dtype=torch.bfloat16),
                            torch.zeros(B, NKV + 1, D, dtype=torch.bfloat16), slots, kc, vc)
    with pytest.raises(ValueError, match="num_tokens"):
        pkv.kv_cache_append(k, k.clone(), slots[:-1], kc, vc)


def test_shared_prefix_calls_check_the_same_shapes():
    q, kc, vc, bt, cl = _decode_args()
    k = torch.zeros(B, NKV, D, dtype=torch.bfloat16)
    slots = torch.zeros(B, dtype=torch.int64)
    with pytest.raises(ValueError, match="k_cache and v_cache"):
        pkv.paged_attention_decode_shared_prefix(q, kc, vc[:-1], bt, cl, prefix_len=16)
    with pytest.raises(ValueError, match="block_tables"):
        pkv.paged_attention_decode_shared_prefix_append(q, k, k.clone(), slots, kc, vc, bt[:-1],
                                                        cl, prefix_len=16)
    with pytest.raises(ValueError, match="block_tables"):
        pkv.paged_attention_decode_noalloc(q, kc, vc, bt[:-1], cl)


def test_block_copy_pools_must_agree():
    kc = torch.zeros(NB, BS, NKV, D, dtype=torch.bfloat16)
    pairs = torch.zeros(1, 2, dtype=torch.int32)
    with pytest.raises(ValueError, match="one shape"):
        pkv.copy_blocks(kc, kc[:-1], kc, kc, pairs)
    with pytest.raises(ValueError, match="differ in size"):
        small = torch.zeros(NB, BS // 2, NKV, D, dtype=torch.bfloat16)
        pkv.copy_blocks(small, small, kc, kc, pairs)
    ks, vs = _scales()
    with pytest.raises(ValueError, match="all four"):
        pkv.copy_blocks(kc, kc, kc, kc, pairs, ks, vs)
    with pytest.raises(ValueError, match="like their caches"):
        pkv.copy_blocks(kc, kc, kc, kc, pairs, ks[:-1], vs[:-1], ks, vs)
    with pytest.raises(TypeError, match="CUDA"):
        pkv.copy_blocks(kc, kc, kc, kc, pairs)


def test_size_queries_refuse_unsupported_dtypes():
    with pytest.raises(TypeError, match="unsupported dtype"):
        pkv.decode_num_splits(4, 8, 128, 4096, torch.float16)
    with pytest.raises(TypeError, match="unsupported dtype"):
        pkv.workspace_size(4, 32, 8, 128, 4096, torch.float16)


# ------------------------------------------------ marshalling, with a fake library

class _FakeLib:
    """Stands in for libpkv.so: records each call's arguments, returns 0 (OK)."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, args))
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    from paged_kv_cache_439_b200 import _native, api
    lib = _FakeLib()
    monkeypatch.setattr(_native, "lib", lambda: lib)
    monkeypatch.setattr(api, "_device", lambda t: 0)
    monkeypatch.setattr(api, "_ptr", lambda t, dev=None: None if t is None else t.data_ptr())
    monkeypatch.setattr(api, "_on", lambda dev, fn, *args: fn(*args))
    monkeypatch.setattr(api, "_stream", lambda stream, dev=None: 0)
    return lib


_CACHE_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "i8": torch.int8,
             "fp8": torch.float8_e4m3fn}


def _cpu_cache(wl):
    shape = (wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim)
    kc = torch.zeros(shape, dtype=torch.int8).view(_CACHE_DT[wl.cache_dtype])
    if wl.cache_dtype not in ("i8", "fp8"):
        kc = torch.zeros(shape, dtype=_CACHE_DT[wl.cache_dtype])
    ks = vs = None
    if wl.cache_dtype in ("i8", "fp8"):
        ks = torch.ones(wl.num_blocks, wl.num_kv_heads, wl.block_size)
        vs = torch.ones_like(ks)
    return kc, kc.clone(), ks, vs


@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8", "f32"])
def test_binding_passes_the_workload_sizes(fake, cache_dtype):
    """Every call of the binding accepts a workload's own tensors and passes the
    library the sizes those tensors have."""
    from paged_kv_cache_439_b200.workloads import make_custom
    wl = make_custom("bind", [5, 40, 17], 8, 2, 64, 16, cache_dtype, seed=3,
                     input_dtype=torch.float32 if cache_dtype == "f32" else torch.bfloat16,
                     shared_prefix=0)
    kc, vc, ks, vs = _cpu_cache(wl)
    err = torch.zeros(1, dtype=torch.int32)
    B, nq, nkv, d = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    nb, bs, maxb = wl.num_blocks, wl.block_size, wl.block_tables.shape[1]
    pkv.kv_cache_append(wl.prefill_k, wl.prefill_v, wl.prefill_slots, kc, vc, ks, vs,
                        err_flag=err)
    name, a = fake.calls[-1]
    assert name == "pkv_kv_cache_append"
    assert a[3:6] == (wl.prefill_k.shape[0], nkv, d) and a[10:12] == (nb, bs)
    ws = torch.empty(256, dtype=torch.float32)
    out = pkv.paged_attention_decode(wl.q, kc, vc, wl.block_tables, wl.context_lens,
                                     k_scale=ks, v_scale=vs, workspace=ws, num_splits=2,
                                     err_flag=err)
    name, a = fake.calls[-1]
    assert name == "pkv_paged_attention_decode" and out.shape == wl.q.shape
    assert a[9] == maxb and a[11] == maxb * bs and a[12:18] == (B, nq, nkv, d, bs, nb)
    assert a[20] == 256 * 4 and a[21] == 2          # workspace bytes, not elements
    if cache_dtype != "f32":
        pkv.paged_attention_decode_append(wl.q, wl.new_k, wl.new_v, wl.new_slots, kc, vc,
                                          wl.block_tables, wl.context_lens, k_scale=ks,
                                          v_scale=vs, err_flag=err)
        name, a = fake.calls[-1]
        assert name == "pkv_paged_attention_decode_append"
        assert a[15:21] == (B, nq, nkv, d, bs, nb)
    pkv.paged_attention_decode_noalloc(wl.q, kc, vc, wl.block_tables, wl.context_lens,
                                       k_scale=ks, v_scale=vs, err_flag=err)
    name, a = fake.calls[-1]
    assert name == "pkv_paged_attention_decode_noalloc" and a[12:18] == (B, nq, nkv, d, bs, nb)


def test_binding_passes_shared_prefix_sizes(fake):
    from paged_kv_cache_439_b200.workloads import make_custom
    wl = make_custom("bind-sp", [200, 150, 160], 8, 2, 128, 16, "bf16", seed=4,
                     shared_prefix=128)
    kc, vc, _, _ = _cpu_cache(wl)
    B, nq, nkv, d = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    pkv.paged_attention_decode_shared_prefix(wl.q, kc, vc, wl.block_tables, wl.context_lens,
                                             128)
    name, a = fake.calls[-1]
    assert name == "pkv_paged_attention_decode_shared_prefix" and a[12:16] == (B, nq, nkv, d)
    assert a[19] == 128
    pkv.paged_attention_decode_shared_prefix_append(wl.q, wl.new_k, wl.new_v, wl.new_slots, kc,
                                                    vc, wl.block_tables, wl.context_lens, 128)
    name, a = fake.calls[-1]
    assert name == "pkv_paged_attention_decode_shared_prefix_append"
    assert a[13:17] == (B, nq, nkv, d) and a[20] == 128


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without libpkv.so every call raises: there is no fallback path."""
    from paged_kv_cache_439_b200 import _native
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "libpkv.so"))
    with pytest.raises(ImportError, match="libpkv.so not found"):
        pkv.decode_num_splits(4, 8, 128, 4096, torch.bfloat16)
    with pytest.raises(ImportError, match="libpkv.so not found"):
        pkv.workspace_size(4, 32, 8, 128, 4096, torch.bfloat16)
    with pytest.raises(ImportError, match="libpkv.so not found"):
        pkv.BlockManager(16, 16)
